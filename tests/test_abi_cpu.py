"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/hkv.h declares, and sizes/validates configs."""
import ctypes as C
import subprocess

import pytest
import torch

import kv_cache_compression_hkv_b200 as hkv
from kv_cache_compression_hkv_b200 import build
from kv_cache_compression_hkv_b200.inputs import WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def test_exports_every_declared_symbol():
    names = hkv.declared_symbols()
    assert len(names) >= 15
    L = hkv.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.check_output(["nm", "-D", "--defined-only", hkv.LIB_PATH], text=True)
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported
    # nothing but the C ABI is exported
    assert all(s.startswith("hkv_") or s.startswith("_") for s in exported), exported - set(names)


def test_status_strings():
    L = hkv.lib()
    for code, name in hkv._lib.STATUS.items():
        assert L.hkv_status_string(code).decode() == name


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_pool_bytes_for_every_workload(name):
    w = WORKLOADS[name]
    for mode in (hkv.MODE_HEADKV, hkv.MODE_FULL):
        n = hkv.pool_bytes(hkv.config_for(w, mode=mode))
        kv = 2 * w.num_layers * w.num_seqs * w.head_dim * (2 if w.dtype == "bf16" else 4)
        H, L = w.num_heads, w.max_len
        T = H * L * w.rho[0] // w.rho[1]
        slots = T + H * w.ste_m if mode == hkv.MODE_HEADKV else H * L
        assert n >= kv * slots
        assert n < kv * slots * 1.6 + (64 << 20)
    assert hkv.pool_bytes(hkv.config_for(w)) < hkv.pool_bytes(hkv.config_for(w, mode=hkv.MODE_FULL))


def test_config_validation():
    base = hkv.config_for(WORKLOADS["llamagen_xl"])
    bad = [dict(num_heads=0), dict(num_heads=33), dict(head_dim=96), dict(ste_m=31), dict(ste_m=0),
           dict(score_window=0), dict(score_window=40), dict(rho_num=2, rho_den=1), dict(tau=0.0),
           dict(tau=1.5), dict(mode=7), dict(stratified=2), dict(max_len=1), dict(max_len=9000),
           dict(local_window=0), dict(cls_queries=-1), dict(cls_queries=9),
           dict(cfg_pairing=3), dict(cfg_pairing=-1), dict(num_seqs=63, cfg_pairing=1),
           dict(num_seqs=63, cfg_pairing=2), dict(heads_total=19), dict(heads_total=5000),
           dict(heads_total=-1),
           dict(rho_num=1, rho_den=64)]  # last: budget below H*W
    for kw in bad:
        cfg = hkv.Config(**{**base.__dict__, **kw})
        with pytest.raises(hkv.HkvError) as e:
            hkv.pool_bytes(cfg)
        assert e.value.code == 1, kw


def test_classifier_variants_accepted():
    base = hkv.config_for(WORKLOADS["llamagen_xl"])
    n = hkv.pool_bytes(base)
    for kw in (dict(cls_queries=0), dict(cls_queries=8), dict(cfg_pairing=hkv.CFG_HALVES),
               dict(cfg_pairing=hkv.CFG_ADJACENT, cls_queries=8), dict(num_seqs=63)):
        assert hkv.pool_bytes(hkv.Config(**{**base.__dict__, **kw})) > 0, kw
    # the variants change no buffer
    assert hkv.pool_bytes(hkv.Config(**{**base.__dict__, "cls_queries": 8, "cfg_pairing": 1})) == n


def test_sharded_heads_pool():
    """A context holding 7 of 20 heads: the budget counts all 20 heads, the
    pool only this shard's slots (T + 7 * M per (sequence, layer))."""
    w = WORKLOADS["llamagen_xl"]
    base = hkv.config_for(w)
    part = hkv.Config(**{**base.__dict__, "num_heads": 7, "heads_total": 20})
    assert hkv.pool_bytes(part) < hkv.pool_bytes(base)
    same = hkv.Config(**{**base.__dict__, "heads_total": 20})
    assert hkv.pool_bytes(same) == hkv.pool_bytes(base)
    for name in ("hkv_prefill_label", "hkv_prefill_compress"):
        assert name in hkv.declared_symbols()


def test_create_rejects_bad_pool_without_touching_the_device():
    cfg = hkv.config_for(WORKLOADS["llamagen_1layer_f32"])
    cc = cfg.c()
    ctx = C.c_void_p()
    L = hkv.lib()
    assert L.hkv_create(C.byref(cc), None, 1 << 20, None, C.byref(ctx)) == 1   # null pool
    assert L.hkv_create(C.byref(cc), 0x1001, 1 << 30, None, C.byref(ctx)) == 1  # misaligned
    assert L.hkv_create(C.byref(cc), 0x100000, 16, None, C.byref(ctx)) == 3  # too small
    assert L.hkv_prefill_classify(None, 0, None, None, None, 10, 640, None, None) == 1
    assert L.hkv_ste_evict(None, 0, 1, None) == 1
    assert L.hkv_ste_select_batch(None, None, None, None, 1, 8, 4, 1, 1, 1, None, None) == 1
    assert L.hkv_prefill_label(None, 0, None, None, None, 10, 640, None, None, None) == 1
    assert L.hkv_prefill_compress(None, 0, None, None, 10, 640, None, None) == 1
    assert L.hkv_classify_groups(None, 4, 8, 1, 40, None, 28, 0.9, None, None, None) == 1
    # nq above r, r above n: rejected before anything is read
    assert L.hkv_classify_groups(0x1000, 4, 8, 9, 40, None, 28, 0.9, 0x2000, 0x3000, None) == 1
    assert L.hkv_classify_groups(0x1000, 4, 8, 8, 7, None, 28, 0.9, 0x2000, 0x3000, None) == 1
    assert L.hkv_classify_groups(0x1000, 0, 8, 8, 40, None, 28, 0.9, 0x2000, 0x3000, None) == 0


def test_create_reports_a_failed_cuda_call():
    """With no CUDA device (this host) a create whose arguments are all
    valid fails in its first runtime call: HKV_ERR_CUDA, no context, and
    nothing written through the pool pointer.  Only where no GPU is visible:
    on a GPU the fake pool address would be handed to the device."""
    if torch.cuda.is_available():
        pytest.skip("needs a host without a visible CUDA device")
    cfg = hkv.config_for(WORKLOADS["llamagen_1layer_f32"])
    cc = cfg.c()
    ctx = C.c_void_p()
    n = hkv.pool_bytes(cfg)
    assert hkv.lib().hkv_create(C.byref(cc), 0x100000, n, None, C.byref(ctx)) == 5
    assert not ctx.value


def test_missing_library_fails_loudly(monkeypatch):
    """No silent fallback: without libhkv.so every entry point raises."""
    from kv_cache_compression_hkv_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/libhkv.so")
    with pytest.raises(RuntimeError, match="libhkv.so not found"):
        _lib.lib()
    with pytest.raises(RuntimeError, match="libhkv.so not found"):
        hkv.pool_bytes(hkv.config_for(WORKLOADS["llamagen_xl"]))
