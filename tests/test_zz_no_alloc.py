"""The allocation-free entry point against the context-based one and the
oracle.

hkv_prefill_classify_noalloc serves callers that cannot allocate device
memory (not even the pool hkv_create needs): during a global-mode graph
capture, under a caching allocator that owns all device memory, or in a
process that may not allocate after start-up.  Its scratch is a fixed array
inside the library, shared by every call.  This file is collected last so a
run that stops at the first failure has run every other test first; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_hkv_b200 as hkv
from kv_cache_compression_hkv_b200 import _lib
from kv_cache_compression_hkv_b200.inputs import WORKLOADS, generate_layer
from oracle import hkv_oracle as O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def built():
    from kv_cache_compression_hkv_b200 import build
    build.build()
    assert torch.cuda.is_available(), "this test needs a CUDA device"


def _context_reference(w, q, k, v):
    """The existing entry point: prefill + grouping through a context."""
    P = w.prefill_len
    cache = hkv.HeadKVCache(hkv.config_for(w, num_layers=1), device=DEV)
    out = torch.empty(w.num_seqs, w.num_heads, P, w.head_dim, dtype=w.torch_dtype, device=DEV)
    cache.prefill_classify(0, q[:, :, :P], k[:, :, :P], v[:, :, :P], out=out)
    lab, ntau = cache.labels(0)
    assert cache.check()[0] == 0
    return out, lab.reshape(-1), ntau.reshape(-1)


@pytest.mark.parametrize("name", ["janus_pro_7b_rho6", "llamagen_1layer_f32"])
def test_noalloc_matches_context_path_two_calls(name):
    w = WORKLOADS[name].scaled(num_layers=1)
    if w.num_seqs > 4:
        w = w.scaled(num_seqs=4)
    P = w.prefill_len
    tol = 1e-5 if w.dtype == "f32" else 2e-2
    for call, seed in enumerate((101, 202)):  # two calls in a row on the shared scratch
        q, k, v = generate_layer(w, 0, seed, DEV)
        ref_out, ref_lab, ref_ntau = _context_reference(w, q, k, v)
        out = torch.empty_like(ref_out)
        n_tau, label, status = _lib.prefill_classify_noalloc(
            q[:, :, :P], k[:, :, :P], v[:, :, :P], w.local_window, 0.9, out=out)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0], call
        np.testing.assert_array_equal(label.cpu().numpy(), ref_lab, err_msg=f"call {call}")
        np.testing.assert_array_equal(n_tau.cpu().numpy(), ref_ntau, err_msg=f"call {call}")
        err = (out.double() - ref_out.double()).abs().max() / ref_out.double().abs().max()
        assert float(err) <= tol, (call, float(err))
        _check_against_oracle(w, q, k, v, out, n_tau, label, tol)


def _check_against_oracle(w, q, k, v, out, n_tau, label, tol):
    """Every block against the oracle's causal attention and grouping of
    the last query's weights on the same bits: outputs within tol, labels
    equal unless the sum of the W-1 newest weights lies within 1e-5 of tau,
    n_tau equal unless a running sum next to the boundary does."""
    P, W = w.prefill_len, w.local_window
    S, H = q.shape[0], q.shape[1]
    got_out = out.double().cpu().numpy().reshape(S, H, P, -1)
    nt, lab = n_tau.cpu().numpy().reshape(S, H), label.cpu().numpy().reshape(S, H)
    for s in range(S):
        for h in range(H):
            qq, kk, vv = (x[s, h, :P].double().cpu().numpy() for x in (q, k, v))
            o, p = O.causal_attention(qq, kk, vv)
            err = np.abs(got_out[s, h] - o).max() / np.abs(o).max()
            assert err <= tol, (s, h, err)
            e_nt, e_lab, cw = O.classify(p[-1], W, 0.9)
            if abs(cw - 0.9) > 1e-5:
                assert lab[s, h] == e_lab, (s, h, cw)
            c = np.cumsum(p[-1][::-1])
            near = [abs(c[i] - 0.9) <= 1e-5 for i in (e_nt - 2, e_nt - 1) if 0 <= i < P]
            if not any(near):
                assert nt[s, h] == e_nt, (s, h)


def test_noalloc_rejects_sizes_beyond_its_array():
    x = torch.zeros(1, 16, 64, dtype=torch.bfloat16, device=DEV)
    n_tau = torch.empty(1, dtype=torch.int32, device=DEV)
    label = torch.empty(1, dtype=torch.uint8, device=DEV)
    too_many_blocks = 2_097_088 // 16 + 1
    rc = _lib.lib().hkv_prefill_classify_noalloc(
        hkv.DTYPE_BF16, 64, too_many_blocks, x.data_ptr(), x.data_ptr(), x.data_ptr(), 16, 16 * 64,
        8, 0.9, None, n_tau.data_ptr(), label.data_ptr(), None, None)
    assert rc == 3  # HKV_ERR_CAPACITY, nothing enqueued
    # the fp32 path's shared memory bounds its prefill length
    xf = torch.zeros(1, 16, 64, dtype=torch.float32, device=DEV)
    P = 12289
    rc = _lib.lib().hkv_prefill_classify_noalloc(
        hkv.DTYPE_F32, 64, 1, xf.data_ptr(), xf.data_ptr(), xf.data_ptr(), P, P * 64,
        8, 0.9, None, n_tau.data_ptr(), label.data_ptr(), None, None)
    assert rc == 1  # HKV_ERR_INVALID_ARG, nothing enqueued
