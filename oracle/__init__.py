"""ctypes front of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module; the library package never does.

``Oracle(path)`` wraps one build of the oracle (the tests also build deliberately
broken copies of ``oracle.c`` and load them through the same class).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile ``source`` with gcc (fp64, OpenMP, no fast-math) into ``output``."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    tmp = output + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


_dptr = ctypes.POINTER(ctypes.c_double)
_bptr = ctypes.POINTER(ctypes.c_ubyte)


def _as_ptr(a: np.ndarray):
    return a.ctypes.data_as(_dptr)


class Oracle:
    """fp64 reference for attention forward (O, LSE) and backward (dQ, dK, dV)."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = build()
        self.lib = ctypes.CDLL(path)
        L = ctypes.c_long
        D, U64 = ctypes.c_double, ctypes.c_ulonglong
        lp = ctypes.POINTER(ctypes.c_long)
        self.lib.oracle_attention_fwd.argtypes = [
            _dptr, _dptr, _dptr, L, L, L, L, D, ctypes.c_int, L, L, _dptr, _bptr, lp, D, U64,
            U64, _dptr, _dptr]
        self.lib.oracle_attention_fwd.restype = ctypes.c_int
        self.lib.oracle_attention_bwd.argtypes = [
            _dptr, _dptr, _dptr, _dptr, L, L, L, L, D, ctypes.c_int, L, L, _dptr, _bptr, lp, D,
            U64, U64, _dptr, _dptr, _dptr]
        self.lib.oracle_attention_bwd.restype = ctypes.c_int
        u32p = ctypes.POINTER(ctypes.c_uint32)
        self.lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        self.lib.oracle_philox4x32_10.restype = None
        self.lib.oracle_dropout_mask.argtypes = [U64, U64, L, L, D, _bptr]
        self.lib.oracle_dropout_mask.restype = ctypes.c_int
        self.lib.oracle_num_threads.restype = ctypes.c_int

    @staticmethod
    def _prep(*arrays):
        out = []
        shape = arrays[0].shape
        for a in arrays:
            a = np.ascontiguousarray(a, dtype=np.float64)
            if a.shape != shape or a.ndim != 4:
                raise ValueError("oracle inputs must share one (B, H, N, d) shape")
            out.append(a)
        return out

    @staticmethod
    def _slopes(alibi, H):
        if alibi is None:
            return None, None
        a = np.ascontiguousarray(alibi, dtype=np.float64).reshape(-1)
        if a.shape != (H,):
            raise ValueError("alibi_slopes must hold one slope per head")
        return a, _as_ptr(a)

    @staticmethod
    def _padding(key_padding, B, N):
        if key_padding is None:
            return None, None
        a = np.ascontiguousarray(key_padding, dtype=np.uint8)
        if a.shape != (B, N):
            raise ValueError("key_padding must be a (B, N) array of flags")
        return a, a.ctypes.data_as(_bptr)

    @staticmethod
    def _lengths(lengths, B, N):
        if lengths is None:
            return None, None
        a = np.ascontiguousarray(lengths, dtype=np.int64).reshape(-1)
        if a.shape != (B,) or np.any(a < 0) or np.any(a > N):
            raise ValueError("lengths must hold one length in [0, N] per batch entry")
        return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_long))

    @staticmethod
    def _dropout(dropout):
        if dropout is None:
            return 0.0, 0, 0
        p, seed, offset = dropout
        return float(p), int(seed), int(offset)

    def philox4x32_10(self, counter, key):
        """The four output words of Philox4x32-10 for a 4-word counter and 2-word key."""
        c = (ctypes.c_uint32 * 4)(*counter)
        k = (ctypes.c_uint32 * 2)(*key)
        out = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, k, out)
        return [int(x) for x in out]

    def dropout_mask(self, seed, offset, bh, N, p):
        """The (N, N) keep flags (query, key) of head bh (= b * H + h)."""
        m = np.empty((N, N), dtype=np.uint8)
        rc = self.lib.oracle_dropout_mask(int(seed), int(offset), int(bh), int(N), float(p),
                                          m.ctypes.data_as(_bptr))
        if rc != 0:
            raise ValueError("dropout probability out of range")
        return m

    def fwd(self, q, k, v, scale, causal=False, window=(-1, -1), alibi=None, key_padding=None,
            dropout=None, lengths=None):
        """Returns (O, LSE) in fp64 for (B, H, N, d) inputs; `alibi`: H slopes or None;
        `key_padding`: (B, N) flags, True for a padded key, or None; `dropout`:
        (p, seed, offset) or None; `lengths`: B real lengths or None."""
        q, k, v = self._prep(q, k, v)
        B, H, N, d = q.shape
        o = np.empty_like(q)
        lse = np.empty((B, H, N), dtype=np.float64)
        keep, slopes = self._slopes(alibi, H)
        keep_pad, pad = self._padding(key_padding, B, N)
        dp, seed, offset = self._dropout(dropout)
        keep_len, lens = self._lengths(lengths, B, N)
        rc = self.lib.oracle_attention_fwd(_as_ptr(q), _as_ptr(k), _as_ptr(v), B, H, N, d,
                                           float(scale), int(bool(causal)), int(window[0]),
                                           int(window[1]), slopes, pad, lens, dp, seed, offset,
                                           _as_ptr(o), _as_ptr(lse))
        if rc != 0:
            raise RuntimeError("oracle_attention_fwd failed with %d" % rc)
        return o, lse

    def bwd(self, q, k, v, do, scale, causal=False, window=(-1, -1), alibi=None,
            key_padding=None, dropout=None, lengths=None):
        """Returns (dQ, dK, dV) in fp64: the gradient of <O, dO> for (B, H, N, d) inputs."""
        q, k, v, do = self._prep(q, k, v, do)
        B, H, N, d = q.shape
        dq = np.empty_like(q)
        dk = np.empty_like(q)
        dv = np.empty_like(q)
        keep, slopes = self._slopes(alibi, H)
        keep_pad, pad = self._padding(key_padding, B, N)
        dp, seed, offset = self._dropout(dropout)
        keep_len, lens = self._lengths(lengths, B, N)
        rc = self.lib.oracle_attention_bwd(_as_ptr(q), _as_ptr(k), _as_ptr(v), _as_ptr(do),
                                           B, H, N, d, float(scale), int(bool(causal)),
                                           int(window[0]), int(window[1]), slopes, pad, lens,
                                           dp, seed, offset, _as_ptr(dq), _as_ptr(dk),
                                           _as_ptr(dv))
        if rc != 0:
            raise RuntimeError("oracle_attention_bwd failed with %d" % rc)
        return dq, dk, dv

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())


_default = None


def default() -> Oracle:
    """The oracle built from ``oracle.c`` in this directory (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def fwd(*args, **kw):
    return default().fwd(*args, **kw)


def bwd(*args, **kw):
    return default().bwd(*args, **kw)
