"""fp64 CPU oracle for SegmentAttention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product path never does.

The arithmetic lives in ``seg_attn_oracle.c`` (plain two-pass softmax
attention in double precision that walks the segment lists itself) and
``seg_la_oracle.c`` (the simple-GLA linear-attention recurrence, token by
token); this file compiles them with gcc on first use and marshals arguments
through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "seg_attn_oracle.c")
_SRC_LA = os.path.join(_HERE, "seg_la_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_libs = {}


def build(force: bool = False, mutant: int = 0) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, OpenMP, IEEE double).

    ``mutant`` > 0 builds a copy with one planted mistake (see the C source),
    used only by the tests that check the pins catch such mistakes."""
    path = _LIB if mutant == 0 else os.path.join(_HERE, f"liboracle_mut{mutant}.so")
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_LA))
    if force or not os.path.exists(path) or os.path.getmtime(path) < newest:
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               f"-DORACLE_MUTANT={mutant}", "-o", tmp, _SRC, _SRC_LA, "-lm"])
        os.replace(tmp, path)
    return path


def _load(mutant: int = 0):
    with _lock:
        if mutant not in _libs:
            lib = ctypes.CDLL(build(mutant=mutant))
            P = ctypes.c_void_p
            lib.oracle_rows.argtypes = [ctypes.c_int, P, P, P, P, P, P, P, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                        ctypes.c_int64, P, P, P, P]
            lib.oracle_rows.restype = ctypes.c_int
            lib.oracle_attention.argtypes = [ctypes.c_int, P, P, P, P, P, P, P, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                             ctypes.c_int, P, P]
            lib.oracle_attention.restype = ctypes.c_int
            lib.oracle_rows_fp8.argtypes = [ctypes.c_int, P, P, P, P, P, P, P, P, P,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_int64, P, P, P,
                                            P]
            lib.oracle_rows_fp8.restype = ctypes.c_int
            lib.oracle_e4m3_decode.argtypes = [P, ctypes.c_int64, P]
            lib.oracle_e4m3_decode.restype = None
            lib.oracle_la.argtypes = [ctypes.c_int, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_double, P, ctypes.c_int64, P, P, P]
            lib.oracle_la.restype = ctypes.c_int
            _libs[mutant] = lib
    return _libs[mutant]


def _i32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32).reshape(-1))


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a.size else ctypes.c_void_p(0)


def attention(q_lens, seg_starts, seg_lens, q, k_pool, v_pool, scale, causal, rows=None,
              mutant=0):
    """Oracle outputs for one batch.

    ``seg_starts`` / ``seg_lens`` are per-request lists (logical order).
    ``q`` is bf16 [sum q_lens, Hq, d]; pools are bf16 [S, Hkv, d] (CPU tensors).
    ``rows``: optional (token_index int64 array, head int32 array); when given,
    only those rows are computed and out is [n, d], lse [n].
    Otherwise out is [sum q_lens, Hq, d] and lse [sum q_lens, Hq].  float64.
    """
    lib = _load(mutant)
    counts = _i32([len(s) for s in seg_starts])
    starts = _i32([x for s in seg_starts for x in s])
    lens = _i32([x for s in seg_lens for x in s])
    ql = _i32(q_lens)
    qb, kb, vb = _bits(q), _bits(k_pool), _bits(v_pool)
    hq, d = q.shape[1], q.shape[2]
    hkv = k_pool.shape[1]
    batch = len(q_lens)
    if rows is None:
        total = int(ql.sum())
        out = np.zeros((total, hq, d), dtype=np.float64)
        lse = np.zeros((total, hq), dtype=np.float64)
        rc = lib.oracle_attention(batch, _ptr(ql), _ptr(counts), _ptr(starts), _ptr(lens),
                                  _ptr(qb), _ptr(kb), _ptr(vb), hq, hkv, d, float(scale),
                                  int(bool(causal)), _ptr(out), _ptr(lse))
    else:
        tok = np.ascontiguousarray(np.asarray(rows[0], dtype=np.int64))
        head = np.ascontiguousarray(np.asarray(rows[1], dtype=np.int32))
        out = np.zeros((tok.size, d), dtype=np.float64)
        lse = np.zeros((tok.size,), dtype=np.float64)
        rc = lib.oracle_rows(batch, _ptr(ql), _ptr(counts), _ptr(starts), _ptr(lens), _ptr(qb),
                             _ptr(kb), _ptr(vb), hq, hkv, d, float(scale), int(bool(causal)),
                             tok.size, _ptr(tok), _ptr(head), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return torch.from_numpy(out), torch.from_numpy(lse)


def batch_attention(wl, batch, rows=None):
    """Convenience wrapper over a synthetic workload's batch."""
    return attention(batch.q_lens, batch.seg_starts, batch.seg_lens, batch.q, wl.k_pool,
                     wl.v_pool, wl.scale, batch.causal, rows=rows)


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of E4M3 codes (uint8 array), from the format definition."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8).reshape(-1))
    out = np.zeros(c.size, dtype=np.float64)
    _load().oracle_e4m3_decode(_ptr(c), c.size, _ptr(out))
    return out


def _codes(t: torch.Tensor) -> np.ndarray:
    assert t.dtype in (torch.uint8, torch.float8_e4m3fn)
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def attention_fp8(q_lens, seg_starts, seg_lens, q, k_pool, v_pool, k_scale, v_scale, scale,
                  causal, rows=None):
    """Oracle for an FP8 (E4M3) KV cache: pools of E4M3 codes with per-kv-head scales
    (``k_scale``/``v_scale``, length Hkv); queries bf16.  Same outputs as ``attention``."""
    lib = _load()
    counts = _i32([len(s) for s in seg_starts])
    starts = _i32([x for s in seg_starts for x in s])
    lens = _i32([x for s in seg_lens for x in s])
    ql = _i32(q_lens)
    qb, kb, vb = _bits(q), _codes(k_pool), _codes(v_pool)
    ks = np.ascontiguousarray(np.asarray(k_scale, dtype=np.float64).reshape(-1))
    vs = np.ascontiguousarray(np.asarray(v_scale, dtype=np.float64).reshape(-1))
    hq, d = q.shape[1], q.shape[2]
    hkv = k_pool.shape[1]
    if rows is None:
        total = int(ql.sum())
        tok = np.repeat(np.arange(total, dtype=np.int64), hq)
        head = np.tile(np.arange(hq, dtype=np.int32), total)
    else:
        tok = np.ascontiguousarray(np.asarray(rows[0], dtype=np.int64))
        head = np.ascontiguousarray(np.asarray(rows[1], dtype=np.int32))
    out = np.zeros((tok.size, d), dtype=np.float64)
    lse = np.zeros((tok.size,), dtype=np.float64)
    rc = lib.oracle_rows_fp8(len(q_lens), _ptr(ql), _ptr(counts), _ptr(starts), _ptr(lens),
                             _ptr(qb), _ptr(kb), _ptr(vb), _ptr(ks), _ptr(vs), hq, hkv, d,
                             float(scale), int(bool(causal)), tok.size, _ptr(tok), _ptr(head),
                             _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    o, l = torch.from_numpy(out), torch.from_numpy(lse)
    if rows is None:
        o, l = o.view(-1, hq, d), l.view(-1, hq)
    return o, l


def linear_attention(q_lens, q, k, v, g, scale, state_in=None, in_slot=None, mutant=0):
    """Oracle of segment linear attention (simple GLA) for one batch.

    ``q, k, v`` bf16 [T, H, d] (CPU), ``g`` [T, H] log-decays (any float dtype, taken as
    float64), ``state_in`` [N, H, d, d] states of the pool (or None), ``in_slot`` per
    request (-1 or None: zero initial state).  Returns (out [T, H, d], state [B, H, d, d])
    in float64."""
    lib = _load(mutant)
    ql = _i32(q_lens)
    batch = ql.size
    T, H, d = q.shape
    slots = _i32(in_slot if in_slot is not None else [-1] * batch)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    gd = np.ascontiguousarray(g.detach().cpu().double().numpy().reshape(-1))
    if state_in is not None:
        st = np.ascontiguousarray(state_in.detach().cpu().double().numpy())
        n_in = st.shape[0]
    else:
        st, n_in = np.zeros(1), 0
    out = np.zeros((T, H, d), dtype=np.float64)
    state = np.zeros((batch, H, d, d), dtype=np.float64)
    rc = lib.oracle_la(batch, _ptr(ql), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(gd), H, d,
                       float(scale), _ptr(st) if n_in else ctypes.c_void_p(0), n_in, _ptr(slots),
                       _ptr(out), _ptr(state))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return torch.from_numpy(out), torch.from_numpy(state)
