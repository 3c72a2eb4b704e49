"""ctypes binding of libhkv (include/hkv.h): argument marshalling only.

Every step of the hot path runs in the library's CUDA kernels; this module
turns torch tensors into pointers, strides and streams, and status codes into
exceptions.  It fails loudly when the library is missing: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhkv.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "hkv.h")

DTYPE_F32, DTYPE_BF16 = 0, 1
MODE_HEADKV, MODE_FULL, MODE_UNIFORM = 0, 1, 2
CFG_UNTIED, CFG_HALVES, CFG_ADJACENT = 0, 1, 2
STATUS = {0: "HKV_OK", 1: "HKV_ERR_INVALID_ARG", 2: "HKV_ERR_STATE", 3: "HKV_ERR_CAPACITY",
          4: "HKV_ERR_NUMERIC", 5: "HKV_ERR_CUDA", 6: "HKV_ERR_TIMEOUT"}


class HkvError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class _Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "num_seqs", "num_layers", "num_heads", "head_dim", "dtype", "max_len", "local_window",
        "ste_m", "near_dist", "score_window", "rho_num", "rho_den", "mode", "stratified",
        "cls_queries", "cfg_pairing", "heads_total")] + [("tau", C.c_double)]


_lib = None


def lib():
    """The loaded libhkv; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libhkv.so not found at {LIB_PATH}; build it with "
                "`python -m kv_cache_compression_hkv_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, I, I64, D, Z = C.c_void_p, C.c_int32, C.c_int64, C.c_double, C.c_size_t
        sig = {
            "hkv_pool_bytes": [P, P],
            "hkv_create": [P, P, Z, P, P],
            "hkv_prefill_classify": [P, I, P, P, P, I, I64, P, P],
            "hkv_prefill_label": [P, I, P, P, P, I, I64, P, P, P],
            "hkv_prefill_compress": [P, I, P, P, I, I64, P, P],
            "hkv_append": [P, I, P, P, P],
            "hkv_decode_attend": [P, I, P, P, P],
            "hkv_decode_step": [P, I, P, P, P, P, P],
            "hkv_ste_evict": [P, I, I, P],
            "hkv_get_labels": [P, I, P, P, P],
            "hkv_get_lens": [P, I, P, P, P],
            "hkv_get_kept": [P, I, I, I, P, I, P, P],
            "hkv_check": [P, P, P],
            "hkv_get_evict_stats": [P, P, P],
            "hkv_clear_error": [P, P],
            "hkv_reset": [P, P],
            "hkv_classify_rows": [P, I, I, I, D, P, P, P],
            "hkv_classify_groups": [P, I, I, I, I, P, I, D, P, P, P],
            "hkv_ste_select_batch": [P, P, P, P, I, I, I, I, I, I, P, P],
            "hkv_prefill_classify_noalloc": [I, I, I, P, P, P, I, I64, I, D, P, P, P, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = C.c_int
        L.hkv_status_string.argtypes = [C.c_int]
        L.hkv_status_string.restype = C.c_char_p
        L.hkv_destroy.argtypes = [P]
        L.hkv_destroy.restype = None
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Function names include/hkv.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(hkv_[a-z_]+)\s*\(", text)))


def _check(rc: int, what: str):
    if rc != 0:
        raise HkvError(rc, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclass
class Config:
    num_seqs: int
    num_layers: int
    num_heads: int
    head_dim: int
    max_len: int
    local_window: int
    ste_m: int
    near_dist: int
    score_window: int = 8
    rho_num: int = 1
    rho_den: int = 4
    dtype: int = DTYPE_BF16
    mode: int = MODE_HEADKV
    stratified: int = 1
    cls_queries: int = 1   # grouping by the last n prefill queries' per-distance weights
    cfg_pairing: int = CFG_UNTIED
    heads_total: int = 0   # heads of a whole (sequence, layer) when heads are sharded
    tau: float = 0.9

    def c(self) -> _Config:
        return _Config(self.num_seqs, self.num_layers, self.num_heads, self.head_dim, self.dtype,
                       self.max_len, self.local_window, self.ste_m, self.near_dist,
                       self.score_window, self.rho_num, self.rho_den, self.mode,
                       int(self.stratified), int(self.cls_queries), int(self.cfg_pairing),
                       int(self.heads_total), float(self.tau))

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == DTYPE_F32 else torch.bfloat16


def pool_bytes(cfg: Config) -> int:
    n = C.c_size_t()
    cc = cfg.c()
    _check(lib().hkv_pool_bytes(C.byref(cc), C.byref(n)), "hkv_pool_bytes")
    return n.value


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


class HeadKVCache:
    """One context of libhkv: a head-aware compressed KV cache for every
    (sequence, layer, head), held in one caller-owned device pool."""

    def __init__(self, cfg: Config, device=None, stream=None):
        self.cfg = cfg
        self.device = torch.device(device if device is not None else "cuda")
        self.nbytes = pool_bytes(cfg)
        self.pool = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
        self._cc = cfg.c()
        ctx = C.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib().hkv_create(C.byref(self._cc), self.pool.data_ptr(), self.nbytes,
                                    _stream(stream), C.byref(ctx)), "hkv_create")
        self.ctx = ctx

    def close(self):
        if getattr(self, "ctx", None) and self.ctx.value:
            lib().hkv_destroy(self.ctx)
            self.ctx = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self, stream=None):
        """Starts a new generation on the same pool (every layer must be
        prefilled and classified again)."""
        _check(lib().hkv_reset(self.ctx, _stream(stream)), "hkv_reset")

    # -- argument checks (shapes, dtypes, devices) ---------------------------
    def _tensor(self, x: torch.Tensor, name: str):
        if not isinstance(x, torch.Tensor) or x.device != self.device or \
                x.dtype != self.cfg.torch_dtype:
            raise ValueError(f"{name}: expected a {self.cfg.torch_dtype} tensor on {self.device}")

    def _step_tensor(self, x: torch.Tensor, name: str):
        self._tensor(x, name)
        c = self.cfg
        if tuple(x.shape) != (c.num_seqs, c.num_heads, c.head_dim) or not x.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous [S, H, d] tensor")

    def _prefill_inputs(self, q, k, v, out):
        c = self.cfg
        for x, nm in ((q, "q"), (k, "k"), (v, "v")):
            self._tensor(x, nm)
            if x.dim() != 4 or x.shape[0] != c.num_seqs or x.shape[1] != c.num_heads or \
                    x.shape[3] != c.head_dim:
                raise ValueError(f"{nm}: expected [S, H, P, d]")
            st = x.stride()
            if st[3] != 1 or st[2] != c.head_dim or st[0] != c.num_heads * st[1]:
                raise ValueError(f"{nm}: unsupported strides {st}")
        if not (q.stride() == k.stride() == v.stride()) or not (q.shape == k.shape == v.shape):
            raise ValueError("q, k, v must share shape and strides")
        P = q.shape[2]
        if out is not None:
            self._tensor(out, "out")
            if tuple(out.shape) != tuple(q.shape) or not out.is_contiguous():
                raise ValueError("out: expected a contiguous [S, H, P, d] tensor")
        return P

    def prefill_classify(self, layer: int, q, k, v, out=None, stream=None):
        """q, k, v: [S, H, P, d] with unit stride in d, stride d in P and the
        (s, h) blocks evenly spaced (a [S, H, L, d] tensor sliced to P works)."""
        P = self._prefill_inputs(q, k, v, out)
        _check(lib().hkv_prefill_classify(self.ctx, layer, q.data_ptr(), k.data_ptr(),
                                          v.data_ptr(), P, q.stride(1), _ptr(out),
                                          _stream(stream)), "hkv_prefill_classify")

    def prefill_label(self, layer: int, q, k, v, out=None, n_local=None, stream=None):
        """Sharded heads, phase 1: prefill attention and grouping of the
        heads held here.  Returns n_local (int32 [S] on the device): each
        sequence's Local count here, to be summed over the shards."""
        P = self._prefill_inputs(q, k, v, out)
        if n_local is None:
            n_local = torch.empty(self.cfg.num_seqs, dtype=torch.int32, device=self.device)
        elif n_local.dtype != torch.int32 or n_local.device != self.device or \
                n_local.numel() != self.cfg.num_seqs or not n_local.is_contiguous():
            raise ValueError("n_local: expected a contiguous int32 [S] tensor on the device")
        _check(lib().hkv_prefill_label(self.ctx, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       P, q.stride(1), _ptr(out), n_local.data_ptr(),
                                       _stream(stream)), "hkv_prefill_label")
        return n_local

    def prefill_compress(self, layer: int, k, v, n_local_total, stream=None):
        """Sharded heads, phase 2: budgets from the all-shards Local counts
        (int32 [S] on the device), then compression at classification.  k, v:
        the same prefill tensors prefill_label got."""
        P = self._prefill_inputs(k, k, v, None)
        t = n_local_total
        if t.dtype != torch.int32 or t.device != self.device or t.numel() != self.cfg.num_seqs \
                or not t.is_contiguous():
            raise ValueError("n_local_total: expected a contiguous int32 [S] tensor on the device")
        _check(lib().hkv_prefill_compress(self.ctx, layer, k.data_ptr(), v.data_ptr(), P,
                                          k.stride(1), t.data_ptr(), _stream(stream)),
               "hkv_prefill_compress")

    def append(self, layer: int, k_t, v_t, stream=None):
        self._step_tensor(k_t, "k_t")
        self._step_tensor(v_t, "v_t")
        _check(lib().hkv_append(self.ctx, layer, k_t.data_ptr(), v_t.data_ptr(), _stream(stream)),
               "hkv_append")

    def decode_attend(self, layer: int, q_t, o_t, stream=None):
        self._step_tensor(q_t, "q_t")
        self._step_tensor(o_t, "o_t")
        _check(lib().hkv_decode_attend(self.ctx, layer, q_t.data_ptr(), o_t.data_ptr(),
                                       _stream(stream)), "hkv_decode_attend")

    def decode_step(self, layer: int, q_t, k_t, v_t, o_t, stream=None):
        for x, nm in ((q_t, "q_t"), (k_t, "k_t"), (v_t, "v_t"), (o_t, "o_t")):
            self._step_tensor(x, nm)
        _check(lib().hkv_decode_step(self.ctx, layer, q_t.data_ptr(), k_t.data_ptr(),
                                     v_t.data_ptr(), o_t.data_ptr(), _stream(stream)),
               "hkv_decode_step")

    def ste_evict(self, layer_begin: int = 0, layer_end: int | None = None, stream=None):
        le = self.cfg.num_layers if layer_end is None else layer_end
        _check(lib().hkv_ste_evict(self.ctx, layer_begin, le, _stream(stream)), "hkv_ste_evict")

    # -- state read-back (synchronises the stream) ---------------------------
    def labels(self, layer: int, stream=None):
        c = self.cfg
        lab = np.zeros((c.num_seqs, c.num_heads), np.uint8)
        nt = np.zeros((c.num_seqs, c.num_heads), np.int32)
        _check(lib().hkv_get_labels(self.ctx, layer, lab.ctypes.data, nt.ctypes.data,
                                    _stream(stream)), "hkv_get_labels")
        return lab, nt

    def lens(self, layer: int, stream=None):
        c = self.cfg
        ln = np.zeros((c.num_seqs, c.num_heads), np.int32)
        bd = np.zeros((c.num_seqs, c.num_heads), np.int32)
        _check(lib().hkv_get_lens(self.ctx, layer, ln.ctypes.data, bd.ctypes.data,
                                  _stream(stream)), "hkv_get_lens")
        return ln, bd

    def kept(self, seq: int, layer: int, head: int, stream=None) -> np.ndarray:
        cap = self.cfg.max_len
        buf = np.zeros(cap, np.int32)
        n = C.c_int32()
        _check(lib().hkv_get_kept(self.ctx, seq, layer, head, buf.ctypes.data, cap, C.byref(n),
                                  _stream(stream)), "hkv_get_kept")
        return buf[: n.value].copy()

    def evict_stats(self, stream=None) -> dict:
        """Evictions since create/reset: heads, tokens scored, rows moved."""
        out = np.zeros(3, dtype=np.int64)
        _check(lib().hkv_get_evict_stats(self.ctx, out.ctypes.data, _stream(stream)),
               "hkv_get_evict_stats")
        return {"heads": int(out[0]), "tokens": int(out[1]), "rows_moved": int(out[2])}

    def check(self, stream=None):
        detail = C.c_int32()
        rc = lib().hkv_check(self.ctx, C.byref(detail), _stream(stream))
        return rc, detail.value

    def clear_error(self, stream=None):
        _check(lib().hkv_clear_error(self.ctx, _stream(stream)), "hkv_clear_error")


def classify_groups(rows: torch.Tensor, nq: int, W: int, tau: float = 0.9, partner=None,
                    stream=None):
    """Grouping of [U, r, n] fp32 kept weight rows (row q: the query at
    position n - r + q) by the mean of the last nq queries' per-distance
    weights, units u and partner[u] (int32 [U], optional) tied.  Returns
    (n_tau int32 [U], label uint8 [U]) on the rows' device."""
    if rows.dtype != torch.float32 or rows.dim() != 3 or not rows.is_cuda or \
            not rows.is_contiguous():
        raise ValueError("rows: expected a contiguous float32 [U, r, n] CUDA tensor")
    U, r, n = rows.shape
    if partner is not None and (partner.dtype != torch.int32 or partner.numel() != U or
                                partner.device != rows.device or not partner.is_contiguous()):
        raise ValueError("partner: expected a contiguous int32 [U] tensor on the rows' device")
    n_tau = torch.empty(U, dtype=torch.int32, device=rows.device)
    label = torch.empty(U, dtype=torch.uint8, device=rows.device)
    _check(lib().hkv_classify_groups(rows.data_ptr(), U, r, nq, n, _ptr(partner), W, float(tau),
                                     n_tau.data_ptr(), label.data_ptr(), _stream(stream)),
           "hkv_classify_groups")
    return n_tau, label


def classify_rows(rows: torch.Tensor, W: int, tau: float = 0.9, stream=None):
    """Grouping rule on fp32 weight rows [n_rows, n] (device); returns
    (n_tau int32, label uint8) device tensors."""
    if rows.dtype != torch.float32 or rows.dim() != 2 or not rows.is_contiguous() or not rows.is_cuda:
        raise ValueError("rows: expected a contiguous fp32 [n_rows, n] CUDA tensor")
    nr, n = rows.shape
    n_tau = torch.empty(nr, dtype=torch.int32, device=rows.device)
    label = torch.empty(nr, dtype=torch.uint8, device=rows.device)
    _check(lib().hkv_classify_rows(rows.data_ptr(), nr, n, W, float(tau), n_tau.data_ptr(),
                                   label.data_ptr(), _stream(stream)), "hkv_classify_rows")
    return n_tau, label


def ste_select_batch(score: torch.Tensor, pos: torch.Tensor, count: torch.Tensor, t: torch.Tensor,
                     D: int, k_near: int, k_far: int, stratified: bool = True, stream=None):
    """Stratified selection on [n_probs, n] fp32 scores / int32 positions
    (device); returns a uint8 evict mask of the same shape."""
    n_probs, n = score.shape
    for x, dt in ((score, torch.float32), (pos, torch.int32), (count, torch.int32), (t, torch.int32)):
        if x.dtype != dt or not x.is_contiguous() or not x.is_cuda:
            raise ValueError("ste_select_batch: bad tensor")
    ev = torch.empty(n_probs, n, dtype=torch.uint8, device=score.device)
    _check(lib().hkv_ste_select_batch(score.data_ptr(), pos.data_ptr(), count.data_ptr(),
                                      t.data_ptr(), n_probs, n, D, k_near, k_far, int(stratified),
                                      ev.data_ptr(), _stream(stream)), "hkv_ste_select_batch")
    return ev


def prefill_classify_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, local_window: int,
                             tau: float = 0.9, out: torch.Tensor | None = None, stream=None):
    """Prefill attention + head grouping with no device allocation by the
    library (see hkv_prefill_classify_noalloc).  q, k, v: [..., P, d] blocks
    with unit stride in d, stride d in P and evenly spaced blocks.  Returns
    (n_tau int32, label uint8, status int32[2]) device tensors; the caller's
    tensors here are the outputs it passes."""
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q, k, v: float32 or bfloat16 only")
    d, P = q.shape[-1], q.shape[-2]
    nb = q.numel() // (P * d) if q.is_contiguous() else int(np.prod(q.shape[:-2]))
    for x in (q, k, v):
        if not x.is_cuda or x.device != q.device or x.dtype != q.dtype:
            raise ValueError("q, k, v: CUDA tensors of one dtype on one device")
        if x.stride(-1) != 1 or x.stride(-2) != d or x.shape != q.shape or x.stride() != q.stride():
            raise ValueError("q, k, v: unsupported layout")
    if out is not None and (out.dtype != q.dtype or out.device != q.device or
                            not out.is_contiguous() or out.numel() != nb * P * d):
        raise ValueError("out: a contiguous tensor of q's dtype and device with n_blocks*P*d elements")
    bs = q.stride(-3) if q.dim() >= 3 else P * d
    if q.dim() == 4 and q.stride(0) != q.shape[1] * q.stride(1):
        raise ValueError("q, k, v: blocks must be evenly spaced")
    dt = DTYPE_F32 if q.dtype == torch.float32 else DTYPE_BF16
    n_tau = torch.empty(nb, dtype=torch.int32, device=q.device)
    label = torch.empty(nb, dtype=torch.uint8, device=q.device)
    status = torch.empty(2, dtype=torch.int32, device=q.device)
    _check(lib().hkv_prefill_classify_noalloc(dt, d, nb, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              P, bs, local_window, float(tau), _ptr(out),
                                              n_tau.data_ptr(), label.data_ptr(), status.data_ptr(),
                                              _stream(stream)), "hkv_prefill_classify_noalloc")
    return n_tau, label, status
