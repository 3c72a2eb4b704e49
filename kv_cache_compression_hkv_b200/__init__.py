"""B200-native head-aware KV-cache compression (HeadKV) for autoregressive
image generation: Python binding of libhkv (include/hkv.h).

The hot path (prefill attention, head grouping, compression, per-step
append + decode attention with fused STE logits, Stratified Token Eviction)
runs in hand-written sm_100a CUDA kernels; this package only marshals
arguments.
"""
from ._lib import (  # noqa: F401
    CFG_ADJACENT, CFG_HALVES, CFG_UNTIED, DTYPE_BF16, DTYPE_F32, MODE_FULL, MODE_HEADKV,
    MODE_UNIFORM, Config, HeadKVCache, HkvError,
    LIB_PATH, classify_groups, classify_rows, declared_symbols, lib, pool_bytes,
    ste_select_batch)


def config_for(w, mode: int = MODE_HEADKV, stratified: bool = True, num_seqs: int | None = None,
               num_layers: int | None = None, cls_queries: int = 1,
               cfg_pairing: int = CFG_UNTIED) -> Config:
    """Library config of a synthetic workload (kv_cache_compression_hkv_b200.inputs)."""
    return Config(
        num_seqs=w.num_seqs if num_seqs is None else num_seqs,
        num_layers=w.num_layers if num_layers is None else num_layers,
        num_heads=w.num_heads, head_dim=w.head_dim, max_len=w.max_len,
        local_window=w.local_window, ste_m=w.ste_m, near_dist=w.near_dist,
        score_window=w.score_window, rho_num=w.rho[0], rho_den=w.rho[1],
        dtype=DTYPE_F32 if w.dtype == "f32" else DTYPE_BF16, mode=mode,
        stratified=int(stratified), cls_queries=cls_queries, cfg_pairing=cfg_pairing, tau=0.9)
