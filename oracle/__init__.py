"""ctypes wrapper of the fp64 MAC-Attention oracle (``mac_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it; the CUDA library never does.  It follows page 1 of
"MAC-Attention: a Match-Amend-Complete Scheme for Fast and Accurate Attention
Computation" (the abstract): match on pre-RoPE queries over a short window,
amend a band before the match boundary, complete with fresh attention on the
tail and a numerically stable merge; a miss is plain decode attention.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mac_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile mac_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(C.Structure):
    _fields_ = [("B", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("D", C.c_int),
                ("W", C.c_int), ("band", C.c_int), ("tau", C.c_double), ("rope_theta", C.c_double),
                ("page_size", C.c_int), ("max_seq", C.c_int), ("max_pages_per_seq", C.c_int),
                ("cut_mode", C.c_int), ("per_head", C.c_int), ("ring_bf16", C.c_int)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.c_void_p
            lib.oracle_create.restype = P
            lib.oracle_create.argtypes = [C.POINTER(_Cfg)]
            lib.oracle_free.argtypes = [P]
            lib.oracle_reset.argtypes = [P, C.c_int]
            lib.oracle_set_tau.argtypes = [P, C.c_double]
            lib.oracle_window.restype = C.c_int
            lib.oracle_window.argtypes = [P, C.c_int, P, P, P, P, P]
            lib.oracle_rope.argtypes = [P, C.c_int, C.c_long, C.c_double, P]
            lib.oracle_partial.argtypes = [P, P, P, C.c_int, C.c_long, C.c_long, C.c_long, P, P, P]
            lib.oracle_merge.argtypes = [P, C.c_double, C.c_double, P, C.c_double, C.c_double,
                                         C.c_int, P, P, P]
            lib.oracle_step.restype = C.c_int
            lib.oracle_step.argtypes = [P] * 14
            lib.oracle_match_step.restype = C.c_int
            lib.oracle_match_step.argtypes = [P] * 7
            lib.oracle_num_threads.restype = C.c_int
            _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def rope(q: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate one pre-RoPE query vector (float32 [D]) to position pos, fp64."""
    q = np.ascontiguousarray(q, np.float32)
    out = np.empty(q.shape[-1], np.float64)
    _load().oracle_rope(_p(q), q.shape[-1], int(pos), float(theta), _p(out))
    return out


def partial(qrot: np.ndarray, K: np.ndarray, V: np.ndarray, x: int, y: int):
    """Exact (o, m, l) of one head over keys [x, y) of contiguous bf16 [L, D] K/V."""
    qrot = np.ascontiguousarray(qrot, np.float64)
    K = np.ascontiguousarray(K, np.uint16)
    V = np.ascontiguousarray(V, np.uint16)
    D = qrot.shape[0]
    o = np.empty(D, np.float64)
    m = np.empty(1, np.float64)
    l = np.empty(1, np.float64)
    _load().oracle_partial(_p(qrot), _p(K), _p(V), D, K.shape[0], int(x), int(y), _p(o), _p(m), _p(l))
    return o, float(m[0]), float(l[0])


def merge(a, b):
    """Numerically stable merge of two (o, m, l) states of disjoint key ranges."""
    o1, m1, l1 = a
    o2, m2, l2 = b
    o1 = np.ascontiguousarray(o1, np.float64)
    o2 = np.ascontiguousarray(o2, np.float64)
    D = o1.shape[0]
    o = np.empty(D, np.float64)
    m = np.empty(1, np.float64)
    l = np.empty(1, np.float64)
    _load().oracle_merge(_p(o1), float(m1), float(l1), _p(o2), float(m2), float(l2), D, _p(o), _p(m), _p(l))
    return o, float(m[0]), float(l[0])


class StepResult:
    __slots__ = ("out", "lse", "hit", "match_pos", "d_best", "d_second", "keys_read")

    def __init__(self, out, lse, hit, match_pos, d_best, d_second, keys_read):
        self.out, self.lse, self.hit, self.match_pos = out, lse, hit, match_pos
        self.d_best, self.d_second, self.keys_read = d_best, d_second, keys_read


class Oracle:
    """Stateful fp64 MAC decode oracle: one instance per layer of KV heads."""

    def __init__(self, B, Hq, Hkv, D, W, band, tau, rope_theta, page_size=0, max_seq=0,
                 max_pages_per_seq=0, cut_mode=0, per_head=0, ring_bf16=0):
        self.lib = _load()
        self.cfg = _Cfg(B, Hq, Hkv, D, W, band, float(tau), float(rope_theta), page_size, max_seq,
                        max_pages_per_seq, cut_mode, per_head, ring_bf16)
        self.h = self.lib.oracle_create(C.byref(self.cfg))
        if not self.h:
            raise ValueError("invalid oracle configuration")
        self.B, self.Hq, self.Hkv, self.D, self.W = B, Hq, Hkv, D, W
        self.G = Hq // Hkv
        self.nd = Hkv * (self.G if per_head else 1)  # match decisions per sequence

    @classmethod
    def for_workload(cls, wl, cache, tau=None, band=None, W=None, cut_mode=0, per_head=0, ring_bf16=0):
        return cls(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W if W is None else W, wl.band if band is None else band,
                   wl.tau if tau is None else tau, wl.rope_theta, wl.page_size,
                   cache.max_seq if not cache.paged else 0,
                   cache.block_table.shape[1] if cache.paged else 0, cut_mode, per_head, ring_bf16)

    def __del__(self):
        try:
            if self.h:
                self.lib.oracle_free(self.h)
                self.h = None
        except Exception:
            pass

    def reset(self, b: int) -> None:
        self.lib.oracle_reset(self.h, b)

    def step(self, q_pre, rope_pos, K, V, block_table, seq_lens) -> StepResult:
        q_pre = np.ascontiguousarray(q_pre, np.float32)
        rope_pos = np.ascontiguousarray(rope_pos, np.int32)
        seq_lens = np.ascontiguousarray(seq_lens, np.int32)
        assert K.dtype == np.uint16 and K.flags.c_contiguous and V.flags.c_contiguous
        bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
        U = self.B * self.nd
        out = np.empty((self.B, self.Hq, self.D), np.float64)
        lse = np.empty((self.B, self.Hq), np.float64)
        hit = np.empty(U, np.uint8)
        mpos = np.empty(U, np.int32)
        db = np.empty(U, np.float64)
        ds = np.empty(U, np.float64)
        kr = C.c_long(0)
        rc = self.lib.oracle_step(self.h, _p(q_pre), _p(rope_pos), _p(K), _p(V), _p(bt), _p(seq_lens),
                                  _p(out), _p(lse), _p(hit), _p(mpos), _p(db), _p(ds), C.byref(kr))
        if rc != 0:
            raise ValueError("oracle_step rejected its inputs (rc=%d)" % rc)
        sh = (self.B, self.nd)
        return StepResult(out, lse, hit.reshape(sh), mpos.reshape(sh), db.reshape(sh), ds.reshape(sh), kr.value)

    def match_step(self, q_pre, seq_lens):
        """Match stage only (no attention): (hit, match_pos, d_best, d_second), each
        [B][Hkv] ([B][Hq] with per-head matching)."""
        q_pre = np.ascontiguousarray(q_pre, np.float32)
        seq_lens = np.ascontiguousarray(seq_lens, np.int32)
        U = self.B * self.nd
        hit = np.empty(U, np.uint8)
        mpos = np.empty(U, np.int32)
        db = np.empty(U, np.float64)
        ds = np.empty(U, np.float64)
        rc = self.lib.oracle_match_step(self.h, _p(q_pre), _p(seq_lens), _p(hit), _p(mpos), _p(db), _p(ds))
        if rc != 0:
            raise ValueError("oracle_match_step rejected its inputs (rc=%d)" % rc)
        sh = (self.B, self.nd)
        return hit.reshape(sh), mpos.reshape(sh), db.reshape(sh), ds.reshape(sh)

    def warm_start(self, q_pre, rope_pos, K, V, block_table, seq_lens) -> None:
        """Seed every window from n prefill positions ([warm] in mac_oracle.c): each
        sequence's window is emptied, then the n positions run as steps with
        threshold 0.  q_pre [n][B][Hq][D], rope_pos and seq_lens [n][B]."""
        for b in range(self.B):
            self.reset(b)
        self.lib.oracle_set_tau(self.h, 0.0)
        try:
            for j in range(len(q_pre)):
                self.step(q_pre[j], rope_pos[j], K, V, block_table, seq_lens[j])
        finally:
            self.lib.oracle_set_tau(self.h, self.cfg.tau)

    def window(self, u: int):
        """(q, o, m, l, pos) of unit u's window, oldest first."""
        W = max(self.W, 1)
        q = np.empty((W, self.G, self.D), np.float32)
        o = np.empty((W, self.G, self.D), np.float64)
        m = np.empty((W, self.G), np.float64)
        l = np.empty((W, self.G), np.float64)
        pos = np.empty(W, np.int32)
        n = self.lib.oracle_window(self.h, u, _p(q), _p(o), _p(m), _p(l), _p(pos))
        return q[:n], o[:n], m[:n], l[:n], pos[:n]
