"""Python access to the CPU oracle in hkv_oracle.c.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the bench's
CPU-baseline leg import this module; the product path never does.  It shares
no code with the CUDA library.

Every array crosses as float64 / int32 / uint8; inputs are the exact values of
the bf16 or fp32 data the GPU consumes (widening to double is exact).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hkv_oracle.c")
_SO = os.path.join(_HERE, "libhkv_oracle.so")
_lib = None

MODE_HEADKV, MODE_FULL, MODE_UNIFORM = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE double, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
             "-shared", "-fPIC", "-o", _SO, _SRC, "-lm"])
    return _SO


class _UnitParams(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "num_heads", "head_dim", "max_len", "prefill_len", "local_window", "ste_m",
        "near_dist", "score_window", "rho_num", "rho_den", "mode", "stratified",
        "cls_queries")] + [
        ("tau", C.c_double), ("label_band", C.c_double), ("select_band", C.c_double),
        ("cls_rows", C.c_void_p)]


class _Hints(C.Structure):
    _fields_ = [("labels", C.c_void_p), ("n_events", C.c_int32),
                ("event_step", C.c_void_p), ("kept", C.c_void_p),
                ("kept_stride", C.c_int32)]


class _UnitOut(C.Structure):
    _fields_ = [("labels", C.c_void_p), ("n_tau", C.c_void_p), ("c_window", C.c_void_p),
                ("o_prefill", C.c_void_p), ("o_decode", C.c_void_p),
                ("kept_final", C.c_void_p), ("len_final", C.c_void_p),
                ("max_events", C.c_int32), ("event_step", C.c_void_p),
                ("evicted", C.c_void_p), ("evicted_stride", C.c_int32)] + [
        (n, C.c_int32) for n in (
            "n_local", "budget_g", "cap_g", "n_events", "n_label_ties", "n_label_hard",
            "n_select", "n_select_ties", "n_select_hard", "first_hard_step")] + [
        ("max_label_tie_gap", C.c_double), ("max_select_tie_gap", C.c_double)]


def lib():
    global _lib
    if _lib is None:
        # HKV_ORACLE_SO lets the mutation test load a deliberately broken copy
        alt = os.environ.get("HKV_ORACLE_SO")
        _lib = C.CDLL(alt if alt else build())
        P, I, D = C.c_void_p, C.c_int32, C.c_double
        _lib.hkvo_causal_attention.argtypes = [P, P, P, I, I, I, I, P, P]
        _lib.hkvo_classify.argtypes = [P, I, I, D, P, P, P]
        _lib.hkvo_class_row.argtypes = [P, P, P, I, I, I, P]
        _lib.hkvo_class_row_from_weights.argtypes = [P, I, I, P]
        _lib.hkvo_budgets.argtypes = [P, I, I, I, I, I, P, P, P]
        _lib.hkvo_ste_select.argtypes = [P, P, I, I, I, I, I, I, P, P, P]
        _lib.hkvo_ste_scores.argtypes = [P, P, I, P, I, I, I, P]
        _lib.hkvo_run_unit.argtypes = [P, P, P, P, P, P]
        for f in ("hkvo_causal_attention", "hkvo_classify", "hkvo_class_row",
                  "hkvo_class_row_from_weights", "hkvo_budgets",
                  "hkvo_ste_select", "hkvo_ste_scores", "hkvo_run_unit"):
            getattr(_lib, f).restype = C.c_int
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def causal_attention(q, k, v, q_pos0: int = 0):
    """Outputs [n_q, d] and weights [n_q, n_k] of causal attention."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    nq, d = q.shape
    nk = k.shape[0]
    o = np.zeros((nq, d))
    p = np.zeros((nq, nk))
    _check(lib().hkvo_causal_attention(_p(q), _p(k), _p(v), nq, nk, d, q_pos0, _p(o), _p(p)),
           "causal_attention")
    return o, p


def classify(p_row, W: int, tau: float = 0.9):
    """(n_tau, label 1=Local/0=Global, c_window) for one weight row."""
    p_row = _f64(p_row)
    nt = C.c_int32()
    lab = C.c_uint8()
    cw = C.c_double()
    _check(lib().hkvo_classify(_p(p_row), p_row.size, W, tau, C.byref(nt), C.byref(lab),
                               C.byref(cw)), "classify")
    return nt.value, lab.value, cw.value


def class_row(q, k, v, nq: int = 1):
    """Classification row [P] of one head from its last nq queries (mean of
    the per-distance weights, in the last query's position order).
    q, k, v: [P, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    P, d = q.shape
    row = np.zeros(P)
    _check(lib().hkvo_class_row(_p(q), _p(k), _p(v), P, d, nq, _p(row)), "class_row")
    return row


def class_row_from_weights(w):
    """Classification row [P] from the weights [nq, P] of the last nq
    queries (row k: the query at position P-nq+k)."""
    w = _f64(w)
    nq, P = w.shape
    row = np.zeros(P)
    _check(lib().hkvo_class_row_from_weights(_p(w), P, nq, _p(row)), "class_row_from_weights")
    return row


def budgets(labels, L: int, W: int, rho_num: int, rho_den: int):
    """(n_local, budget_g, total) or ValueError when T < H * W."""
    labels = np.ascontiguousarray(np.asarray(labels, dtype=np.uint8))
    nl, bg, tot = C.c_int32(), C.c_int32(), C.c_int64()
    _check(lib().hkvo_budgets(_p(labels), labels.size, L, W, rho_num, rho_den,
                              C.byref(nl), C.byref(bg), C.byref(tot)), "budgets")
    return nl.value, bg.value, tot.value


def ste_select(score, pos, t: int, D: int, k_near: int, k_far: int, stratified: bool = True):
    """Boolean evict mask plus the near/far boundary gaps."""
    score, pos = _f64(score), _i32(pos)
    ev = np.zeros(score.size, dtype=np.uint8)
    gn, gf = C.c_double(), C.c_double()
    _check(lib().hkvo_ste_select(_p(score), _p(pos), score.size, t, D, k_near, k_far,
                                 int(stratified), _p(ev), C.byref(gn), C.byref(gf)),
           "ste_select")
    return ev.astype(bool), gn.value, gf.value


def ste_scores(q_all, k_all, kept, t: int, r: int):
    q_all, k_all, kept = _f64(q_all), _f64(k_all), _i32(kept)
    s = np.zeros(kept.size)
    _check(lib().hkvo_ste_scores(_p(q_all), _p(k_all), q_all.shape[1], _p(kept), kept.size,
                                 t, r, _p(s)), "ste_scores")
    return s


@dataclass
class UnitParams:
    num_heads: int
    head_dim: int
    max_len: int
    prefill_len: int
    local_window: int
    ste_m: int
    near_dist: int
    score_window: int = 8
    rho_num: int = 1
    rho_den: int = 4
    mode: int = MODE_HEADKV
    stratified: bool = True
    cls_queries: int = 1
    tau: float = 0.9
    label_band: float = 0.0
    select_band: float = 0.0


@dataclass
class UnitResult:
    labels: np.ndarray
    n_tau: np.ndarray
    c_window: np.ndarray
    o_prefill: np.ndarray | None
    o_decode: np.ndarray | None
    kept_final: list
    event_step: np.ndarray
    evicted: np.ndarray
    n_local: int
    budget_g: int
    cap_g: int
    stats: dict = field(default_factory=dict)


def run_unit(prm: UnitParams, q, k, v, hints: dict | None = None,
             want_prefill: bool = False, want_decode: bool = True,
             max_events: int | None = None, cls_rows=None) -> UnitResult:
    """Run one (sequence, layer) unit.  q, k, v: [H, L, d].

    cls_rows (optional): [H, P] classification rows to group by instead of
    the unit's own (labels tied across a CFG pair).

    hints (optional): {"labels": uint8[H], "event_step": int32[E],
    "kept": int32[E, H, stride]} -- another implementation's decisions,
    adopted only where the oracle's own differ by a near-tie (see the bands).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    H, L, d = q.shape
    P = prm.prefill_len
    cp = _UnitParams(H, d, L, P, prm.local_window, prm.ste_m, prm.near_dist,
                     prm.score_window, prm.rho_num, prm.rho_den, prm.mode,
                     int(prm.stratified), prm.cls_queries, prm.tau, prm.label_band,
                     prm.select_band)
    if cls_rows is not None:
        cls_rows = _f64(cls_rows)
        if cls_rows.shape != (H, P):
            raise ValueError("cls_rows must be [H, P]")
        cp.cls_rows = _p(cls_rows).value
    labels = np.zeros(H, np.uint8)
    n_tau = np.zeros(H, np.int32)
    cw = np.zeros(H)
    o_pre = np.zeros((H, P, d)) if want_prefill else None
    o_dec = np.zeros((L - P, H, d)) if want_decode else None
    kept = np.full((H, L), -1, np.int32)
    lens = np.zeros(H, np.int32)
    if max_events is None:
        max_events = (L - P) // 2 + 2
    stride = max(prm.ste_m, P)
    ev_step = np.full(max_events, -1, np.int32)
    evicted = np.full((max_events, H, stride), -1, np.int32)
    out = _UnitOut(_p(labels).value, _p(n_tau).value, _p(cw).value,
                   None if o_pre is None else _p(o_pre).value,
                   None if o_dec is None else _p(o_dec).value,
                   _p(kept).value, _p(lens).value, max_events, _p(ev_step).value,
                   _p(evicted).value, stride)
    hp = None
    keep_alive = []
    if hints is not None:
        hl = None if hints.get("labels") is None else np.ascontiguousarray(
            np.asarray(hints["labels"], np.uint8))
        hs = _i32(hints.get("event_step", np.zeros(0)))
        hk = hints.get("kept")
        hk = None if hk is None else _i32(hk)
        keep_alive += [hl, hs, hk]
        hp = _Hints(None if hl is None else _p(hl).value, hs.size, _p(hs).value,
                    None if hk is None else _p(hk).value,
                    0 if hk is None else hk.shape[-1])
    _check(lib().hkvo_run_unit(C.byref(cp), _p(q), _p(k), _p(v),
                               None if hp is None else C.byref(hp), C.byref(out)),
           "run_unit")
    ne = out.n_events
    return UnitResult(
        labels=labels, n_tau=n_tau, c_window=cw, o_prefill=o_pre, o_decode=o_dec,
        kept_final=[kept[h, :lens[h]].copy() for h in range(H)],
        event_step=ev_step[:min(ne, max_events)],
        evicted=evicted[:min(ne, max_events)],
        n_local=out.n_local, budget_g=out.budget_g, cap_g=out.cap_g,
        stats=dict(n_events=ne, n_label_ties=out.n_label_ties, n_label_hard=out.n_label_hard,
                   n_select=out.n_select, n_select_ties=out.n_select_ties,
                   n_select_hard=out.n_select_hard, first_hard_step=out.first_hard_step,
                   max_label_tie_gap=out.max_label_tie_gap,
                   max_select_tie_gap=out.max_select_tie_gap))


CFG_UNTIED, CFG_HALVES, CFG_ADJACENT = 0, 1, 2


def cfg_partner(s: int, num_seqs: int, pairing: int) -> int:
    """The other sequence of s's classifier-free-guidance pair: the same
    image's conditional and unconditional streams.  CFG_HALVES: the batch
    is [conditional | unconditional], s pairs with s +- S/2; CFG_ADJACENT:
    the two streams alternate, s pairs with s xor 1; CFG_UNTIED: s alone."""
    if pairing == CFG_UNTIED:
        return s
    if num_seqs % 2:
        raise ValueError("CFG pairs need an even number of sequences")
    if pairing == CFG_HALVES:
        half = num_seqs // 2
        return s + half if s < half else s - half
    if pairing == CFG_ADJACENT:
        return s ^ 1
    raise ValueError(f"unknown CFG pairing {pairing}")


def tied_rows(rows_a, rows_b):
    """Classification rows shared by a CFG pair: the plain mean of the two
    sequences' rows, so that both streams of an image get one label per
    (layer, head) and hence the same budgets."""
    return 0.5 * (_f64(rows_a) + _f64(rows_b))
