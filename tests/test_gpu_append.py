"""dsa_cache_append on the GPU against the oracle's cache_append: e4m3 codes, fp32 scales
and copied latent rows are bit-exact; rows no token names keep their contents; tokens with
a bad sequence, position or block-table entry are skipped and reported."""

import numpy as np
import pytest
import torch

from oracle import dsa_ref as R
from sparse_attention_long_03_b200 import dsa

pytestmark = pytest.mark.gpu

PAGE = 64


def _case(rng, D, Dkv, batch=3, max_blocks=4, nb=16, n_valid=200, bad=True):
    k8 = rng.integers(0, 256, (nb * PAGE, D), dtype=np.uint8)  # arbitrary prior contents
    ks = rng.standard_normal(nb * PAGE).astype(np.float32)
    kv = rng.integers(0, 65536, (nb * PAGE, Dkv), dtype=np.uint16)
    bt = rng.permutation(nb).astype(np.int32)[: batch * max_blocks].reshape(batch, max_blocks)
    if bad:
        bt[2, 3] = nb + 5  # a block-table entry out of range
    pairs = rng.choice(batch * max_blocks * PAGE, n_valid, replace=False)
    tok_seq = (pairs // (max_blocks * PAGE)).astype(np.int32)
    tok_pos = (pairs % (max_blocks * PAGE)).astype(np.int32)
    if bad:  # sequence out of range; position past the block table
        tok_seq = np.concatenate([tok_seq, [batch, 0]]).astype(np.int32)
        tok_pos = np.concatenate([tok_pos, [0, max_blocks * PAGE]]).astype(np.int32)
    n = tok_seq.shape[0]
    # keys of very different magnitudes, one all-zero key (scale 1)
    k_in = (rng.standard_normal((n, D)) * rng.uniform(1e-3, 1e3, (n, 1))).astype(np.float32)
    k_in[5] = 0.0
    kv_in = rng.integers(0, 65536, (n, Dkv), dtype=np.uint16)
    return k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


@pytest.mark.parametrize("D,Dkv", [(128, 576), (32, 80)])
def test_append_matches_oracle(D, Dkv):
    rng = np.random.default_rng(D)
    k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in = _case(rng, D, Dkv)
    want8, want_s, want_kv, ok = R.cache_append(k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in)
    assert ok.sum() < len(ok)  # the case does hold bad tokens
    d8, ds, dkv, dbt = _dev(k8), _dev(ks), _dev(kv.view(np.int16)), _dev(bt)
    cache = dsa.make_cache(d8, ds, dkv, dbt)  # holds raw pointers: keep the tensors alive
    dsa.dsa_cache_append(cache, d8, ds, dkv, _dev(tok_seq), _dev(tok_pos), _dev(k_in),
                         _dev(kv_in.view(np.int16)))
    assert dsa.dsa_read_device_status() == 5  # DSA_ERR_BAD_INDEX for the skipped tokens
    assert np.array_equal(d8.cpu().numpy(), want8)
    assert np.array_equal(ds.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    assert np.array_equal(dkv.cpu().numpy().view(np.uint16), want_kv)


def test_append_keys_only_and_status_clean():
    rng = np.random.default_rng(77)
    k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in = _case(rng, 128, 576, bad=False)
    want8, want_s, _, ok = R.cache_append(k8, ks, None, bt, tok_seq, tok_pos, k_in, None)
    assert ok.all()
    d8, ds, dkv, dbt = _dev(k8), _dev(ks), _dev(kv.view(np.int16)), _dev(bt)
    cache = dsa.make_cache(d8, ds, dkv, dbt)  # holds raw pointers: keep the tensors alive
    dsa.dsa_cache_append(cache, d8, ds, None, _dev(tok_seq), _dev(tok_pos), _dev(k_in), None)
    assert dsa.dsa_read_device_status() == 0
    assert np.array_equal(d8.cpu().numpy(), want8)
    assert np.array_equal(ds.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    assert np.array_equal(dkv.cpu().numpy().view(np.uint16), kv)  # latent rows untouched
