"""SegmentAttention for B200: Python binding of the C-ABI library ``libsegattn.so``.

Every function here only marshals arguments for the C entry points declared
in ``include/seg_attn.h`` (same names).  All compute runs in the library's
sm_100a kernels; there is no fallback path.  PyTorch supplies device memory
and streams only.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

from ._build import LIB as LIB_PATH

__all__ = [
    "SegAttnError", "seg_attn_table_desc", "seg_attn_build_table", "seg_attn_workspace_size",
    "seg_attn_prefill", "seg_attn_decode", "seg_attn_status_string", "seg_attn_version",
    "seg_attn_take_device_error", "seg_attn_wait_selftest", "seg_attn_stall_test", "seg_attn_order_test", "SegTable", "load_library", "LIB_PATH",
    "MODE_PREFILL", "MODE_DECODE", "STATUS", "SegPool", "seg_attn_kv_append",
    "seg_attn_decode_fp8", "seg_attn_prefill_fp8", "seg_attn_kv_append_fp8", "SHARE_PREFIX",
    "seg_la_table_desc", "seg_la_build_table", "seg_la_workspace_size", "seg_la_prefill",
    "seg_la_decode", "LATable",
]

MODE_PREFILL = 0
MODE_DECODE = 1
SHARE_PREFIX = 0x100  # OR into the mode: plan shared prefixes
STATUS = {
    "OK": 0, "INVALID_ARG": -1, "SEGMENT_OOB": -2, "SEGMENT_OVERLAP": -3, "QLEN_GT_KLEN": -4,
    "WORKSPACE": -5, "UNSUPPORTED": -6, "CUDA": -7, "BUFFER_TOO_SMALL": -8, "NO_SPACE": -9,
}


class seg_attn_table_desc(ctypes.Structure):
    """Mirror of ``seg_attn_table_desc`` in include/seg_attn.h."""
    _fields_ = [
        ("magic", ctypes.c_uint32), ("version", ctypes.c_uint32),
        ("mode", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("batch", ctypes.c_int32), ("q_heads", ctypes.c_int32),
        ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_slots", ctypes.c_int64), ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("num_segments", ctypes.c_int32), ("num_work", ctypes.c_int32),
        ("queries_per_tile", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
        ("max_k_tiles", ctypes.c_int32), ("num_merge", ctypes.c_int32),
        ("num_parts", ctypes.c_int32), ("shared", ctypes.c_int32),
        ("off_q_offsets", ctypes.c_int64), ("off_k_lens", ctypes.c_int64),
        ("off_seg_offsets", ctypes.c_int64), ("off_seg_start", ctypes.c_int64),
        ("off_seg_kstart", ctypes.c_int64), ("off_seg_len", ctypes.c_int64),
        ("off_work", ctypes.c_int64), ("off_req_chunks", ctypes.c_int64),
        ("off_merge", ctypes.c_int64),
        ("table_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
        ("num_groups", ctypes.c_int32), ("num_group_segments", ctypes.c_int32),
        ("num_group_work", ctypes.c_int32), ("num_group_parts", ctypes.c_int32),
        ("num_citems", ctypes.c_int32), ("num_cascade", ctypes.c_int32),
        ("num_single", ctypes.c_int32), ("num_group_single", ctypes.c_int32),
        ("group_total_k", ctypes.c_int64),
        ("off_group_req", ctypes.c_int64), ("off_group_q_offsets", ctypes.c_int64),
        ("off_group_k_lens", ctypes.c_int64), ("off_group_seg_offsets", ctypes.c_int64),
        ("off_group_seg_start", ctypes.c_int64), ("off_group_seg_kstart", ctypes.c_int64),
        ("off_group_seg_len", ctypes.c_int64), ("off_group_work", ctypes.c_int64),
        ("off_citem", ctypes.c_int64), ("off_cascade", ctypes.c_int64),
    ]


class seg_la_table_desc(ctypes.Structure):
    """Mirror of ``seg_la_table_desc`` in include/seg_la.h."""
    _fields_ = [
        ("magic", ctypes.c_uint32), ("version", ctypes.c_uint32),
        ("mode", ctypes.c_int32), ("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
        ("num_chunks", ctypes.c_int32),
        ("total_q", ctypes.c_int64), ("num_state_slots", ctypes.c_int64),
        ("off_q_offsets", ctypes.c_int64), ("off_in_slot", ctypes.c_int64),
        ("off_out_slot", ctypes.c_int64), ("off_req_chunks", ctypes.c_int64),
        ("off_chunks", ctypes.c_int64),
        ("table_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
    ]


class seg_attn_pool_stats(ctypes.Structure):
    """Mirror of ``seg_attn_pool_stats`` in include/seg_attn.h."""
    _fields_ = [("num_slots", ctypes.c_int64), ("free_slots", ctypes.c_int64),
                ("free_runs", ctypes.c_int64), ("largest_free_run", ctypes.c_int64),
                ("sequences", ctypes.c_int64), ("segments", ctypes.c_int64)]


class SegAttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {seg_attn_status_string(code)} (status {code})")


_lock = threading.Lock()
_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libsegattn.so (built in-tree by ``__graft_entry__.build()``); fail loudly if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = path or LIB_PATH
        if not os.path.exists(path):
            raise ImportError(f"CUDA library not built: {path} is missing "
                              "(run python -c 'import __graft_entry__; __graft_entry__.build()')")
        lib = ctypes.CDLL(path)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(seg_attn_table_desc)
        lib.seg_attn_build_table.argtypes = [I, P, P, P, P, I64, I, I, I, I, I, P, SZ, D]
        lib.seg_attn_build_table.restype = I
        lib.seg_attn_workspace_size.argtypes = [D]
        lib.seg_attn_workspace_size.restype = SZ
        for fn in (lib.seg_attn_prefill, lib.seg_attn_decode):
            fn.argtypes = [P, P, P, P, P, P, D, ctypes.c_float, P, SZ, P]
            fn.restype = I
        lib.seg_attn_status_string.argtypes = [I]
        lib.seg_attn_status_string.restype = ctypes.c_char_p
        lib.seg_attn_version.argtypes = []
        lib.seg_attn_version.restype = I
        lib.seg_attn_take_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
        lib.seg_attn_take_device_error.restype = I
        lib.seg_attn_wait_selftest.argtypes = [I, P]
        lib.seg_attn_wait_selftest.restype = I
        lib.seg_attn_stall_test.argtypes = [I, I]
        lib.seg_attn_stall_test.restype = I
        lib.seg_attn_order_test.argtypes = [I]
        lib.seg_attn_order_test.restype = I
        PP = ctypes.POINTER(ctypes.c_void_p)
        lib.seg_attn_pool_create.argtypes = [I64, PP]
        lib.seg_attn_pool_destroy.argtypes = [P]
        lib.seg_attn_pool_append.argtypes = [P, I64, I64, P]
        lib.seg_attn_pool_release.argtypes = [P, I64]
        lib.seg_attn_pool_segments.argtypes = [P, I64, P, P, I, ctypes.POINTER(I)]
        lib.seg_attn_pool_get_stats.argtypes = [P, ctypes.POINTER(seg_attn_pool_stats)]
        for fn in (lib.seg_attn_pool_create, lib.seg_attn_pool_destroy, lib.seg_attn_pool_append,
                   lib.seg_attn_pool_release, lib.seg_attn_pool_segments,
                   lib.seg_attn_pool_get_stats):
            fn.restype = I
        lib.seg_attn_kv_append.argtypes = [P, P, P, I64, I, I, P, P, I64, P]
        lib.seg_attn_kv_append.restype = I
        lib.seg_attn_kv_append_fp8.argtypes = [P, P, P, I64, I, I, P, P, P, P, I64, P]
        lib.seg_attn_kv_append_fp8.restype = I
        for fn in (lib.seg_attn_decode_fp8, lib.seg_attn_prefill_fp8):
            fn.argtypes = [P, P, P, P, P, P, P, P, D, ctypes.c_float, P, SZ, P]
            fn.restype = I
        LD = ctypes.POINTER(seg_la_table_desc)
        lib.seg_la_build_table.argtypes = [I, P, P, P, I64, I, I, I, P, SZ, LD]
        lib.seg_la_build_table.restype = I
        lib.seg_la_workspace_size.argtypes = [LD]
        lib.seg_la_workspace_size.restype = SZ
        lib.seg_la_prefill.argtypes = [P, P, P, P, P, P, P, LD, ctypes.c_float, P, SZ, P]
        lib.seg_la_prefill.restype = I
        lib.seg_la_decode.argtypes = [P, P, P, P, P, P, P, LD, ctypes.c_float, P]
        lib.seg_la_decode.restype = I
        _lib = lib
        return lib


def seg_attn_status_string(code: int) -> str:
    return load_library().seg_attn_status_string(int(code)).decode()


def seg_attn_version() -> int:
    return load_library().seg_attn_version()


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32).reshape(-1))


def _np_ptr(a: Optional[np.ndarray]):
    return ctypes.c_void_p(a.ctypes.data) if a is not None and a.size else ctypes.c_void_p(0)


def seg_attn_build_table(batch: int, q_lens: Optional[Sequence[int]], seg_counts: Sequence[int],
                         seg_starts: Sequence[int], seg_lens: Sequence[int], num_slots: int,
                         causal: bool, mode: int, q_heads: int, kv_heads: int, head_dim: int,
                         pin: bool = False):
    """Returns (host table as an int32 torch tensor, seg_attn_table_desc).  Raises SegAttnError."""
    lib = load_library()
    ql = _i32(q_lens) if q_lens is not None else None
    sc, ss, sl = _i32(seg_counts), _i32(seg_starts), _i32(seg_lens)
    desc = seg_attn_table_desc()
    args = [int(batch), _np_ptr(ql), _np_ptr(sc), _np_ptr(ss), _np_ptr(sl), int(num_slots),
            int(bool(causal)), int(mode), int(q_heads), int(kv_heads), int(head_dim)]
    rc = lib.seg_attn_build_table(*args, ctypes.c_void_p(0), 0, ctypes.byref(desc))
    if rc != 0:
        raise SegAttnError("seg_attn_build_table", rc)
    n = max(1, (desc.table_bytes + 3) // 4)
    host = torch.zeros(n, dtype=torch.int32, pin_memory=pin)
    rc = lib.seg_attn_build_table(*args, ctypes.c_void_p(host.data_ptr()), int(desc.table_bytes),
                                  ctypes.byref(desc))
    if rc != 0:
        raise SegAttnError("seg_attn_build_table", rc)
    return host, desc


def seg_attn_workspace_size(desc: seg_attn_table_desc) -> int:
    return int(load_library().seg_attn_workspace_size(ctypes.byref(desc)))


def _dptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _compute(fn_name, q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale, workspace,
             stream):
    lib = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = getattr(lib, fn_name)(_dptr(q), _dptr(k_pool), _dptr(v_pool), _dptr(out), _dptr(lse),
                               _dptr(dev_table), ctypes.byref(desc), float(softmax_scale),
                               _dptr(workspace), int(ws_bytes), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError(fn_name, rc)


def seg_attn_prefill(q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
                     workspace=None, stream=None) -> None:
    """Launch chunked-prefill attention on ``stream`` (default: torch's current stream)."""
    _compute("seg_attn_prefill", q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
             workspace, stream)


def seg_attn_decode(q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
                    workspace=None, stream=None) -> None:
    """Launch split-K decode attention on ``stream`` (default: torch's current stream)."""
    _compute("seg_attn_decode", q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
             workspace, stream)


def seg_attn_wait_selftest(wait_us: int, stream=None) -> None:
    """Launch the bounded-wait diagnostic: a wait that nothing completes gives up after
    ``wait_us`` and sets bit 0 of the device error word."""
    rc = load_library().seg_attn_wait_selftest(int(wait_us), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError("seg_attn_wait_selftest", rc)


def seg_attn_stall_test(withhold_k_tile: int, wait_us: int = 1000000) -> None:
    """Stall test switch of later prefill launches: the producer stops before K tile
    ``withhold_k_tile`` (< 0: off) and every bounded wait gives up after ``wait_us``."""
    rc = load_library().seg_attn_stall_test(int(withhold_k_tile), int(wait_us))
    if rc != 0:
        raise SegAttnError("seg_attn_stall_test", rc)


def seg_attn_order_test(delay_ns: int) -> None:
    """Order test switch of later prefill launches: every softmax warp of a one-tile item
    sleeps ``delay_ns`` after signalling P of the item's last K tile (0: off)."""
    rc = load_library().seg_attn_order_test(int(delay_ns))
    if rc != 0:
        raise SegAttnError("seg_attn_order_test", rc)


def seg_attn_take_device_error() -> int:
    v = ctypes.c_int(0)
    rc = load_library().seg_attn_take_device_error(ctypes.byref(v))
    if rc != 0:
        raise SegAttnError("seg_attn_take_device_error", rc)
    return v.value


@dataclass
class SegTable:
    """A built table: host copy, description, device copy and workspace size."""
    host: torch.Tensor
    desc: seg_attn_table_desc
    device: Optional[torch.Tensor] = None

    @classmethod
    def build(cls, q_lens, seg_starts, seg_lens, num_slots, causal, mode, q_heads, kv_heads,
              head_dim, pin=False):
        """Per-request lists in, flattened for seg_attn_build_table."""
        counts = [len(s) for s in seg_starts]
        starts = [x for s in seg_starts for x in s]
        lens = [x for s in seg_lens for x in s]
        host, desc = seg_attn_build_table(len(counts), q_lens, counts, starts, lens, num_slots,
                                          causal, mode, q_heads, kv_heads, head_dim, pin=pin)
        return cls(host=host, desc=desc)

    def to(self, device, non_blocking=False) -> "SegTable":
        self.device = self.host.to(device, non_blocking=non_blocking)
        return self

    @property
    def workspace_bytes(self) -> int:
        return seg_attn_workspace_size(self.desc)


class SegPool:
    """Host segment allocator of a slot pool (wraps the seg_attn_pool_* calls)."""

    def __init__(self, num_slots: int):
        self._lib = load_library()
        self._h = ctypes.c_void_p()
        rc = self._lib.seg_attn_pool_create(int(num_slots), ctypes.byref(self._h))
        if rc != 0:
            raise SegAttnError("seg_attn_pool_create", rc)

    def close(self):
        if self._h:
            self._lib.seg_attn_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def append(self, seq: int, n_tokens: int) -> np.ndarray:
        """Slots (int32, logical order) of n_tokens new tokens of sequence ``seq``."""
        out = np.zeros(max(1, int(n_tokens)), dtype=np.int32)
        rc = self._lib.seg_attn_pool_append(self._h, int(seq), int(n_tokens),
                                            ctypes.c_void_p(out.ctypes.data))
        if rc != 0:
            raise SegAttnError("seg_attn_pool_append", rc)
        return out[:n_tokens]

    def release(self, seq: int) -> None:
        rc = self._lib.seg_attn_pool_release(self._h, int(seq))
        if rc != 0:
            raise SegAttnError("seg_attn_pool_release", rc)

    def segments(self, seq: int):
        """(starts, lens) lists of ``seq`` in logical order."""
        count = ctypes.c_int(0)
        self._lib.seg_attn_pool_segments(self._h, int(seq), None, None, 0, ctypes.byref(count))
        n = count.value
        st = np.zeros(max(1, n), dtype=np.int32)
        ln = np.zeros(max(1, n), dtype=np.int32)
        rc = self._lib.seg_attn_pool_segments(self._h, int(seq), ctypes.c_void_p(st.ctypes.data),
                                              ctypes.c_void_p(ln.ctypes.data), n,
                                              ctypes.byref(count))
        if rc != 0:
            raise SegAttnError("seg_attn_pool_segments", rc)
        return st[:n].tolist(), ln[:n].tolist()

    def stats(self) -> dict:
        st = seg_attn_pool_stats()
        rc = self._lib.seg_attn_pool_get_stats(self._h, ctypes.byref(st))
        if rc != 0:
            raise SegAttnError("seg_attn_pool_get_stats", rc)
        return {name: getattr(st, name) for name, _ in st._fields_}


def seg_attn_kv_append(k_new, v_new, slots, k_pool, v_pool, stream=None) -> None:
    """Write k_new / v_new [n, Hkv, d] (device bf16) into the pools at ``slots`` (device int32)."""
    lib = load_library()
    rc = lib.seg_attn_kv_append(_dptr(k_new), _dptr(v_new), _dptr(slots), int(slots.numel()),
                                int(k_pool.shape[1]), int(k_pool.shape[2]), _dptr(k_pool),
                                _dptr(v_pool), int(k_pool.shape[0]), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError("seg_attn_kv_append", rc)


def seg_attn_kv_append_fp8(k_new, v_new, slots, k_scale, v_scale, k_pool, v_pool,
                           stream=None) -> None:
    """Quantise k_new / v_new (bf16 [n, Hkv, d]) with per-kv-head scales and write the E4M3
    codes into uint8 pools [S, Hkv, d] at ``slots``."""
    lib = load_library()
    rc = lib.seg_attn_kv_append_fp8(_dptr(k_new), _dptr(v_new), _dptr(slots), int(slots.numel()),
                                    int(k_pool.shape[1]), int(k_pool.shape[2]), _dptr(k_scale),
                                    _dptr(v_scale), _dptr(k_pool), _dptr(v_pool),
                                    int(k_pool.shape[0]), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError("seg_attn_kv_append_fp8", rc)


def _compute_fp8(fn_name, q, k_pool, v_pool, k_scale, v_scale, out, lse, dev_table, desc,
                 softmax_scale, workspace, stream):
    lib = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = getattr(lib, fn_name)(_dptr(q), _dptr(k_pool), _dptr(v_pool), _dptr(k_scale),
                               _dptr(v_scale), _dptr(out), _dptr(lse), _dptr(dev_table),
                               ctypes.byref(desc), float(softmax_scale), _dptr(workspace),
                               int(ws_bytes), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError(fn_name, rc)


def seg_attn_decode_fp8(q, k_pool, v_pool, k_scale, v_scale, out, lse, dev_table, desc,
                        softmax_scale, workspace=None, stream=None) -> None:
    """Decode over E4M3 pools (uint8 [S, Hkv, d]) with per-kv-head fp32 scales."""
    _compute_fp8("seg_attn_decode_fp8", q, k_pool, v_pool, k_scale, v_scale, out, lse, dev_table,
                 desc, softmax_scale, workspace, stream)


def seg_attn_prefill_fp8(q, k_pool, v_pool, k_scale, v_scale, out, lse, dev_table, desc,
                         softmax_scale, workspace=None, stream=None) -> None:
    """Chunked prefill over E4M3 pools (uint8 [S, Hkv, d]) with per-kv-head fp32 scales."""
    _compute_fp8("seg_attn_prefill_fp8", q, k_pool, v_pool, k_scale, v_scale, out, lse,
                 dev_table, desc, softmax_scale, workspace, stream)


# ----------------------------------------------------------------- segment linear attention
def seg_la_build_table(q_lens, in_slot, out_slot, num_state_slots: int, mode: int, heads: int,
                       head_dim: int, pin: bool = False):
    """Returns (host table int32 tensor, seg_la_table_desc).  ``q_lens`` may be None in decode
    mode.  Raises SegAttnError."""
    lib = load_library()
    ins, outs = _i32(in_slot), _i32(out_slot)
    ql = _i32(q_lens) if q_lens is not None else None
    desc = seg_la_table_desc()
    args = [int(ins.size), _np_ptr(ql), _np_ptr(ins), _np_ptr(outs), int(num_state_slots),
            int(mode), int(heads), int(head_dim)]
    rc = lib.seg_la_build_table(*args, ctypes.c_void_p(0), 0, ctypes.byref(desc))
    if rc != 0:
        raise SegAttnError("seg_la_build_table", rc)
    host = torch.zeros(max(1, (desc.table_bytes + 3) // 4), dtype=torch.int32, pin_memory=pin)
    rc = lib.seg_la_build_table(*args, ctypes.c_void_p(host.data_ptr()), int(desc.table_bytes),
                                ctypes.byref(desc))
    if rc != 0:
        raise SegAttnError("seg_la_build_table", rc)
    return host, desc


def seg_la_workspace_size(desc: seg_la_table_desc) -> int:
    return int(load_library().seg_la_workspace_size(ctypes.byref(desc)))


def seg_la_prefill(q, k, v, g, out, state_pool, dev_table, desc, scale, workspace=None,
                   stream=None) -> None:
    """Chunked simple-GLA prefill on ``stream`` (default: torch's current stream)."""
    lib = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.seg_la_prefill(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(out), _dptr(state_pool),
                            _dptr(dev_table), ctypes.byref(desc), float(scale), _dptr(workspace),
                            int(ws_bytes), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError("seg_la_prefill", rc)


def seg_la_decode(q, k, v, g, out, state_pool, dev_table, desc, scale, stream=None) -> None:
    """One-token simple-GLA decode on ``stream`` (default: torch's current stream)."""
    lib = load_library()
    rc = lib.seg_la_decode(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(out), _dptr(state_pool),
                           _dptr(dev_table), ctypes.byref(desc), float(scale), _stream_ptr(stream))
    if rc != 0:
        raise SegAttnError("seg_la_decode", rc)


@dataclass
class LATable:
    """A built linear-attention table: host copy, description, device copy."""
    host: torch.Tensor
    desc: seg_la_table_desc
    device: Optional[torch.Tensor] = None

    @classmethod
    def build(cls, q_lens, in_slot, out_slot, num_state_slots, mode, heads, head_dim, pin=False):
        host, desc = seg_la_build_table(q_lens, in_slot, out_slot, num_state_slots, mode, heads,
                                        head_dim, pin=pin)
        return cls(host=host, desc=desc)

    def to(self, device, non_blocking=False) -> "LATable":
        self.device = self.host.to(device, non_blocking=non_blocking)
        return self

    @property
    def workspace_bytes(self) -> int:
        return seg_la_workspace_size(self.desc)
