"""Python binding of libdkv (ctypes): argument marshalling only.

Every operation runs in the CUDA kernels of libdkv.so.  torch tensors carry
device memory and the current CUDA stream; nothing here computes the method.
Importing fails loudly when libdkv.so has not been built.

One block-diffusion layer, in outline (bf16 tensors on the GPU; K, V and the
active block are [B, Hkv, block, 128], queries and output [B, Hq, block, 128]):

    cfg = make_config(B, Hq, Hkv, 128, block, k_bits=4, v_bits=4, k_group=32,
                      v_group=32, max_protected=P, max_tokens=capacity)
    cache = dkv_cache_alloc(cfg)
    for each denoising step of the active block:
        dkv_block_attention(cache, q, k_act, v_act, softmax_scale, out)
    dkv_commit_block(cache, k_block, v_block, protect_words)  # block done
    ...
    flags = dkv_cache_status(cache)     # DKV_FLAG_* raised on the device
    dkv_cache_free(cache)

Variants: dkv_block_attention_dual (a second, suffix cache),
dkv_cache_set_v_rotation (K-RPBH-rotated V, before the first commit),
dkv_block_attention_noalloc (no allocation, for stream capture),
dkv_cache_truncate (roll back to a prefix).
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# DKV_LIB selects another build of the library (the bounds-checking
# libdkv_bc.so, for tests); the default is the in-tree libdkv.so
LIB_PATH = os.environ.get("DKV_LIB") or os.path.join(_HERE, "libdkv.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dkv.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python quantized_kv_cache_dkv_b200/build.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

DKV_OK, DKV_ERR_INVALID_ARG, DKV_ERR_UNSUPPORTED, DKV_ERR_CAPACITY, DKV_ERR_CUDA = 0, 1, 2, 3, 4
DKV_FLAG_CAPACITY, DKV_FLAG_RANGE, DKV_FLAG_TIMEOUT, DKV_FLAG_BOUNDS = 0x1, 0x2, 0x4, 0x8
DKV_OPT_SPLITS, DKV_OPT_ATTN_KERNEL, DKV_OPT_PROFILE, DKV_OPT_TEST_STALL = 1, 2, 3, 4
DKV_KERNEL_ATTENTION, DKV_KERNEL_COMBINE, DKV_KERNEL_COMMIT, DKV_KERNEL_TRUNCATE = 0, 1, 2, 3


class DkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libdkv error {code}: {msg}")
        self.code = code


class dkv_config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("q_heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block", ctypes.c_int32), ("k_bits", ctypes.c_int32),
                ("v_bits", ctypes.c_int32), ("k_group", ctypes.c_int32),
                ("v_group", ctypes.c_int32), ("max_protected", ctypes.c_int32),
                ("max_tokens", ctypes.c_int64), ("sink_tokens", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_P = ctypes.c_void_p


class dkv_export(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("k_codes", "k_sz", "k_raw", "k_tail", "tail_mask", "v_codes",
                                   "v_sz", "v_raw", "prot_count", "prot_pos", "prot_k",
                                   "prot_gstart", "v_sink")]


def _sig(name, args):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = ctypes.c_int
    return f


_lib.dkv_last_error.argtypes = []
_lib.dkv_last_error.restype = ctypes.c_char_p
_alloc = _sig("dkv_cache_alloc", [ctypes.POINTER(dkv_config), _P, ctypes.POINTER(_P)])
_free = _sig("dkv_cache_free", [_P])
_commit = _sig("dkv_commit_block", [_P, _P, _P, _P, _P])
_commit_seqs = _sig("dkv_commit_block_seqs", [_P, _P, _P, _P, _P, ctypes.c_int32, _P])
_seq_lens = _sig("dkv_cache_seq_lens", [_P, _P])
_truncate_seq = _sig("dkv_cache_truncate_seq", [_P, ctypes.c_int32, ctypes.c_int64, _P])
_export_seq = _sig("dkv_cache_export_seq", [_P, ctypes.c_int32, _P, ctypes.POINTER(dkv_export)])
_attn = _sig("dkv_block_attention", [_P, _P, _P, _P, ctypes.c_float, _P, _P])
_attn_sel = _sig("dkv_block_attention_selected", [_P, _P, _P, _P, ctypes.c_float, ctypes.c_int32,
                                                  _P, _P, _P, _P])
_attn_noalloc = _sig("dkv_block_attention_noalloc", [_P, _P, _P, _P, ctypes.c_float, _P, _P])
DKV_NOALLOC_SCRATCH_BYTES = 16 << 20
_len = _sig("dkv_cache_len", [_P, ctypes.POINTER(ctypes.c_int64)])
_truncate = _sig("dkv_cache_truncate", [_P, ctypes.c_int64, _P])
_status = _sig("dkv_cache_status", [_P, _P, ctypes.POINTER(ctypes.c_uint32)])
_export = _sig("dkv_cache_export", [_P, _P, ctypes.POINTER(dkv_export)])
_setopt = _sig("dkv_cache_set_option", [_P, ctypes.c_int32, ctypes.c_int64])
_setrot = _sig("dkv_cache_set_v_rotation", [_P, _P, _P, ctypes.c_int32])
_attn_dual = _sig("dkv_block_attention_dual", [_P, _P, _P, _P, _P, ctypes.c_float, _P, _P])
_prof = _sig("dkv_profile_read", [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_int64)])
_plan = _sig("dkv_last_attention_plan", [_P, ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_int32)])


def _check(rc: int) -> None:
    if rc != DKV_OK:
        raise DkvError(rc, (_lib.dkv_last_error() or b"").decode())


def header_symbols() -> list:
    """Names of the functions include/dkv.h declares."""
    txt = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(dkv_\w+)\s*\(", txt, re.M)))


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def make_config(B, Hq, Hkv, d=128, blk=32, k_bits=4, v_bits=4, k_group=32, v_group=32,
                max_protected=0, max_tokens=1024, sink_tokens=0) -> dkv_config:
    return dkv_config(B, Hq, Hkv, d, blk, k_bits, v_bits, k_group, v_group, max_protected,
                      max_tokens, sink_tokens, 0)


class Cache:
    """Owns one dkv_cache handle (freed on close / garbage collection)."""

    def __init__(self, cfg: dkv_config, stream=None):
        self.cfg = cfg
        h = _P()
        _check(_alloc(ctypes.byref(cfg), _stream(stream), ctypes.byref(h)))
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            _check(_free(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def units(self):
        return self.cfg.batch * self.cfg.kv_heads


def _tensor_check(t, shape, name, dtypes):
    if t.device.type != "cuda" or not t.is_contiguous() or tuple(t.shape) != tuple(shape) \
            or t.dtype not in dtypes:
        raise ValueError(f"{name}: need a contiguous CUDA tensor of shape {tuple(shape)} "
                         f"and dtype in {dtypes}, got {tuple(t.shape)} {t.dtype} on {t.device}")


def dkv_cache_alloc(cfg: dkv_config, stream=None) -> Cache:
    return Cache(cfg, stream)


def dkv_cache_free(cache: Cache) -> None:
    cache.close()


def dkv_commit_block(cache: Cache, k, v, protect_words=None, stream=None) -> None:
    import torch
    c = cache.cfg
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k, shp, "k", (torch.bfloat16, torch.int16))
    _tensor_check(v, shp, "v", (torch.bfloat16, torch.int16))
    if protect_words is not None:
        _tensor_check(protect_words, (c.batch, c.kv_heads, c.block // 32), "protect_words",
                      (torch.int32,))
    _check(_commit(cache.h, _ptr(k), _ptr(v), _ptr(protect_words), _stream(stream)))


def dkv_commit_block_seqs(cache: Cache, k, v, protect_words=None, seqs=(), stream=None) -> None:
    """Commit one block to the listed sequences only (each at its own
    length); shapes as in dkv_commit_block, other sequences' rows unread."""
    import torch
    c = cache.cfg
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k, shp, "k", (torch.bfloat16, torch.int16))
    _tensor_check(v, shp, "v", (torch.bfloat16, torch.int16))
    if protect_words is not None:
        _tensor_check(protect_words, (c.batch, c.kv_heads, c.block // 32), "protect_words",
                      (torch.int32,))
    s = np.ascontiguousarray(np.asarray(list(seqs), dtype=np.int32))
    _check(_commit_seqs(cache.h, _ptr(k), _ptr(v), _ptr(protect_words),
                        s.ctypes.data_as(_P) if s.size else None, int(s.size), _stream(stream)))


def dkv_cache_seq_lens(cache: Cache) -> list:
    out = np.zeros(cache.cfg.batch, np.int64)
    _check(_seq_lens(cache.h, out.ctypes.data_as(_P)))
    return [int(x) for x in out]


def dkv_cache_truncate_seq(cache: Cache, seq: int, new_len: int, stream=None) -> None:
    _check(_truncate_seq(cache.h, int(seq), int(new_len), _stream(stream)))


def dkv_block_attention(cache: Cache, q, k_act, v_act, softmax_scale: float, out,
                        stream=None) -> None:
    import torch
    c = cache.cfg
    _tensor_check(q, (c.batch, c.q_heads, c.block, c.head_dim), "q", (torch.bfloat16, torch.int16))
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k_act, shp, "k_act", (torch.bfloat16, torch.int16))
    _tensor_check(v_act, shp, "v_act", (torch.bfloat16, torch.int16))
    _tensor_check(out, (c.batch, c.q_heads, c.block, c.head_dim), "out",
                  (torch.bfloat16, torch.int16))
    _check(_attn(cache.h, _ptr(q), _ptr(k_act), _ptr(v_act), ctypes.c_float(softmax_scale),
                 _ptr(out), _stream(stream)))


def dkv_block_attention_selected(cache: Cache, q, k_act, v_act, softmax_scale: float,
                                 budget: int, out, selected=None, scores=None,
                                 stream=None) -> None:
    """Q-MaskAhead selection: attention over the `budget` committed tokens
    of largest contribution score per (sequence, kv-head) plus the active
    block.  selected: int32 [B, Hkv, budget] or None (the kept positions,
    ascending, -1 after them); scores: float32 [B, Hkv, max_tokens] or None."""
    import torch
    c = cache.cfg
    _tensor_check(q, (c.batch, c.q_heads, c.block, c.head_dim), "q", (torch.bfloat16, torch.int16))
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k_act, shp, "k_act", (torch.bfloat16, torch.int16))
    _tensor_check(v_act, shp, "v_act", (torch.bfloat16, torch.int16))
    _tensor_check(out, (c.batch, c.q_heads, c.block, c.head_dim), "out",
                  (torch.bfloat16, torch.int16))
    if selected is not None:
        _tensor_check(selected, (c.batch, c.kv_heads, budget), "selected", (torch.int32,))
    if scores is not None:
        _tensor_check(scores, (c.batch, c.kv_heads, c.max_tokens), "scores", (torch.float32,))
    _check(_attn_sel(cache.h, _ptr(q), _ptr(k_act), _ptr(v_act), ctypes.c_float(softmax_scale),
                     int(budget), _ptr(out), _ptr(selected), _ptr(scores), _stream(stream)))


def dkv_block_attention_noalloc(cache: Cache, q, k_act, v_act, softmax_scale: float, out,
                                stream=None) -> None:
    """dkv_block_attention for callers that cannot call cudaMalloc (under CUDA
    stream capture, or inside a host application that owns all device
    memory): split scratch comes from a fixed 16 MiB buffer inside libdkv and
    nothing is allocated.  Calls overlapping on the GPU share that buffer and
    race; the first call on a device should come before any stream capture."""
    import torch
    c = cache.cfg
    _tensor_check(q, (c.batch, c.q_heads, c.block, c.head_dim), "q", (torch.bfloat16, torch.int16))
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k_act, shp, "k_act", (torch.bfloat16, torch.int16))
    _tensor_check(v_act, shp, "v_act", (torch.bfloat16, torch.int16))
    _tensor_check(out, (c.batch, c.q_heads, c.block, c.head_dim), "out",
                  (torch.bfloat16, torch.int16))
    _check(_attn_noalloc(cache.h, _ptr(q), _ptr(k_act), _ptr(v_act),
                         ctypes.c_float(softmax_scale), _ptr(out), _stream(stream)))


def dkv_cache_truncate(cache: Cache, new_len: int, stream=None) -> None:
    _check(_truncate(cache.h, new_len, _stream(stream)))


def dkv_block_attention_dual(prefix: Cache, suffix: Cache, q, k_act, v_act,
                             softmax_scale: float, out, stream=None) -> None:
    """Attention of the active block over prefix cache + active block +
    suffix cache (dual-cache reuse); shapes as in dkv_block_attention."""
    import torch
    c = prefix.cfg
    _tensor_check(q, (c.batch, c.q_heads, c.block, c.head_dim), "q", (torch.bfloat16, torch.int16))
    shp = (c.batch, c.kv_heads, c.block, c.head_dim)
    _tensor_check(k_act, shp, "k_act", (torch.bfloat16, torch.int16))
    _tensor_check(v_act, shp, "v_act", (torch.bfloat16, torch.int16))
    _tensor_check(out, (c.batch, c.q_heads, c.block, c.head_dim), "out",
                  (torch.bfloat16, torch.int16))
    _check(_attn_dual(prefix.h, suffix.h, _ptr(q), _ptr(k_act), _ptr(v_act),
                      ctypes.c_float(softmax_scale), _ptr(out), _stream(stream)))


def dkv_cache_set_v_rotation(cache: Cache, perm=None, mix=None, block: int = 0) -> None:
    """K-RPBH rotation of V (before the first commit): perm int32 [128], a
    permutation; mix float32 [k, k] orthogonal, k = 128 / block; block in
    {16, 32, 64, 128}, or 0 (perm, mix None) to turn the rotation off."""
    import numpy as np
    if block == 0:
        _check(_setrot(cache.h, None, None, 0))
        return
    p = np.ascontiguousarray(perm, dtype=np.int32)
    m = np.ascontiguousarray(mix, dtype=np.float32)
    if p.shape != (128,) or m.shape != (128 // block, 128 // block):
        raise ValueError(f"perm must be [128] and mix [{128 // block}, {128 // block}]")
    _check(_setrot(cache.h, p.ctypes.data_as(_P), m.ctypes.data_as(_P), int(block)))


def dkv_cache_len(cache: Cache) -> int:
    n = ctypes.c_int64()
    _check(_len(cache.h, ctypes.byref(n)))
    return n.value


def dkv_cache_status(cache: Cache, stream=None) -> int:
    f = ctypes.c_uint32()
    _check(_status(cache.h, _stream(stream), ctypes.byref(f)))
    return f.value


def dkv_cache_set_option(cache: Cache, key: int, value: int) -> None:
    _check(_setopt(cache.h, key, value))


def dkv_profile_read(cache: Cache, kind: int):
    """(total device ms, launches) of one kernel kind since the last read."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(_prof(cache.h, kind, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def dkv_last_attention_plan(cache: Cache):
    k, s, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_plan(cache.h, ctypes.byref(k), ctypes.byref(s), ctypes.byref(n)))
    return k.value, s.value, n.value


def dkv_cache_export(cache: Cache, stream=None) -> dict:
    """Canonical host copies of the committed state (numpy arrays)."""
    c = cache.cfg
    return _export_arrays(cache, c.batch * c.kv_heads, dkv_cache_len(cache),
                          lambda e: _export(cache.h, _stream(stream), ctypes.byref(e)))


def dkv_cache_export_seq(cache: Cache, seq: int, stream=None) -> dict:
    """Canonical host copies of one sequence's units at its own length."""
    c = cache.cfg
    return _export_arrays(cache, c.kv_heads, dkv_cache_seq_lens(cache)[seq],
                          lambda e: _export_seq(cache.h, int(seq), _stream(stream), ctypes.byref(e)))


def _export_arrays(cache: Cache, U: int, L: int, call) -> dict:
    c = cache.cfg
    d = c.head_dim
    out = {"len": L}
    if c.k_bits < 16:
        Lq = (L // c.k_group) * c.k_group
        nG = Lq // c.k_group
        out["k_codes"] = np.zeros((U, nG, d, c.k_group * c.k_bits // 32), np.uint32)
        out["k_sz"] = np.zeros((U, nG, d, 2), np.float16)
        out["k_tail"] = np.zeros((U, L - Lq, d), np.uint16)
        out["tail_mask"] = np.zeros((U, (c.k_group + 31) // 32), np.uint32)
        out["prot_gstart"] = np.zeros((U, nG + 1), np.int32)
        out["prot_pos"] = np.zeros((U, c.max_protected), np.int32)
        out["prot_k"] = np.zeros((U, c.max_protected, d), np.uint16)
    else:
        out["k_raw"] = np.zeros((U, L, d), np.uint16)
    out["prot_count"] = np.zeros(U, np.int32)
    if c.v_bits < 16:
        out["v_codes"] = np.zeros((U, L, d * c.v_bits // 32), np.uint32)
        out["v_sz"] = np.zeros((U, L, d // c.v_group, 2), np.float16)
        if c.sink_tokens > 0:
            out["v_sink"] = np.zeros((U, min(c.sink_tokens, L), d), np.uint16)
    else:
        out["v_raw"] = np.zeros((U, L, d), np.uint16)
    e = dkv_export()
    for name, _ in dkv_export._fields_:
        arr = out.get(name)
        if arr is not None and arr.size:
            setattr(e, name, arr.ctypes.data)
    _check(call(e))
    return out
