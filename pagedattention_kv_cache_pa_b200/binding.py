"""ctypes binding of libpa (include/pa.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: torch tensors are checked for dtype / device /
contiguity and passed as raw pointers; the work runs in libpa's kernels.
Importing this module fails loudly if libpa.so has not been built — there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
# PA_LIBRARY points the binding at another build of the same ABI (e.g. a tuning variant)
LIB_PATH = os.environ.get("PA_LIBRARY") or os.path.join(PKG, "libpa.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "pa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError("libpa.so is not built (%s); run __graft_entry__.build() or "
                      "python pagedattention_kv_cache_pa_b200/_build.py" % LIB_PATH)

lib = ctypes.CDLL(LIB_PATH)

PA_OK = 0
STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_CUDA",
          -4: "PA_ERR_WORKSPACE", -5: "PA_ERR_OOM_BLOCKS", -6: "PA_ERR_SHARED_BLOCK",
          -7: "PA_ERR_BAD_BLOCK", -8: "PA_ERR_BAD_LENGTH", -9: "PA_ERR_TIMEOUT"}
PA_KERNEL_AUTO, PA_KERNEL_SIMT, PA_KERNEL_TENSOR, PA_KERNEL_TENSOR_SPLIT = 0, 1, 2, 3
PA_FLAG_CHECK = 1
PA_FLAG_PDL = 2
PA_FLAG_SELFTEST_STALL = 4
PA_KV_BF16 = 0
PA_KV_E4M3 = 1


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, pa_status_string(status)))


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32)]

    @classmethod
    def make(cls, *, num_blocks, block_size, num_kv_heads, num_q_heads, head_dim,
             max_blocks_per_seq) -> "CacheDesc":
        return cls(num_blocks, block_size, num_kv_heads, num_q_heads, head_dim, max_blocks_per_seq)


class DecodeOptions(ctypes.Structure):
    _fields_ = [("split_tokens", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("max_ctas", ctypes.c_int32),
                ("rope_theta", ctypes.c_float), ("kv_dtype", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


class DecodePlanInfo(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("ctas", ctypes.c_int32),
                ("split_tokens", ctypes.c_int32), ("max_splits", ctypes.c_int32)]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_DESC = ctypes.POINTER(CacheDesc)
_OPTS = ctypes.POINTER(DecodeOptions)

lib.pa_status_string.argtypes = [ctypes.c_int]
lib.pa_status_string.restype = ctypes.c_char_p
lib.pa_append_kv.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, _DESC, _vp]
lib.pa_append_kv.restype = ctypes.c_int
lib.pa_rope_append_kv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, ctypes.c_float, _vp, _vp, _DESC,
                                  _vp]
lib.pa_rope_append_kv.restype = ctypes.c_int
lib.pa_decode_workspace_size.argtypes = [_i32, _i32, _DESC]
lib.pa_decode_workspace_size.restype = _sz
lib.pa_decode_workspace_size_ex.argtypes = [_i32, _i32, _DESC, _OPTS]
lib.pa_decode_workspace_size_ex.restype = _sz
lib.pa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp, _sz,
                          _DESC, _vp]
lib.pa_decode.restype = ctypes.c_int
lib.pa_decode_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp, _sz,
                             _DESC, _OPTS, _vp]
lib.pa_decode_ex.restype = ctypes.c_int
lib.pa_append_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp,
                                 _vp, _sz, _DESC, _OPTS, _vp]
lib.pa_append_decode.restype = ctypes.c_int
lib.pa_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _DESC,
                                  _OPTS, _vp]
lib.pa_decode_noalloc.restype = ctypes.c_int
lib.pa_decode_status.argtypes = [_vp, _sz, _vp]
lib.pa_decode_status.restype = ctypes.c_int
lib.pa_decode_max_splits.argtypes = [_i32, _i32, _DESC, _OPTS]
lib.pa_decode_max_splits.restype = _i32
lib.pa_decode_describe.argtypes = [_i32, _i32, _DESC, _OPTS, ctypes.POINTER(DecodePlanInfo)]
lib.pa_decode_describe.restype = ctypes.c_int
lib.pa_slot_mapping.argtypes = [_vp, _i32, _vp, _i32, _i32, _vp]
lib.pa_slot_mapping.restype = ctypes.c_int
lib.pa_bm_create.argtypes = [_i32, _i32, _i32, _i32, _vp, _i32, ctypes.POINTER(_vp)]
lib.pa_bm_create.restype = ctypes.c_int
lib.pa_bm_destroy.argtypes = [_vp]
lib.pa_bm_destroy.restype = None
lib.pa_bm_import_seq.argtypes = [_vp, _i32, _i32, _vp]
lib.pa_bm_import_seq.restype = ctypes.c_int
lib.pa_bm_add_seq.argtypes = [_vp, _i32, _i32]
lib.pa_bm_add_seq.restype = ctypes.c_int
lib.pa_bm_fork_seq.argtypes = [_vp, _i32, _i32, _i32, _i32]
lib.pa_bm_fork_seq.restype = ctypes.c_int
lib.pa_bm_free_seq.argtypes = [_vp, _i32]
lib.pa_bm_free_seq.restype = ctypes.c_int
lib.pa_bm_append_tokens.argtypes = [_vp, _vp, _i32, _vp]
lib.pa_bm_append_tokens.restype = ctypes.c_int
lib.pa_bm_num_free.argtypes = [_vp]
lib.pa_bm_num_free.restype = _i32
lib.pa_bm_refcount.argtypes = [_vp, _i32]
lib.pa_bm_refcount.restype = _i32
lib.pa_bm_block_tables.argtypes = [_vp]
lib.pa_bm_block_tables.restype = ctypes.POINTER(ctypes.c_int32)
lib.pa_bm_context_lens.argtypes = [_vp]
lib.pa_bm_context_lens.restype = ctypes.POINTER(ctypes.c_int32)
lib.pa_bm_take_dirty_rows.argtypes = [_vp, _vp, _i32]
lib.pa_bm_take_dirty_rows.restype = _i32
lib.pa_bm_add_seq_tokens.argtypes = [_vp, _i32, _vp, _i32, _vp]
lib.pa_bm_add_seq_tokens.restype = ctypes.c_int
lib.pa_bm_fork_all.argtypes = [_vp, _i32, _i32]
lib.pa_bm_fork_all.restype = ctypes.c_int
lib.pa_bm_append_token_ids.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, _vp]
lib.pa_bm_append_token_ids.restype = ctypes.c_int
lib.pa_bm_num_cached_blocks.argtypes = [_vp]
lib.pa_bm_num_cached_blocks.restype = _i32
lib.pa_copy_blocks.argtypes = [_vp, _vp, _vp, _i32, _DESC, _vp]
lib.pa_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp, _sz, _DESC, _i32, _vp]
lib.pa_prefill.restype = ctypes.c_int
lib.pa_append_kv_e4m3.argtypes = [_vp, _vp, _vp, _i32, ctypes.c_float, ctypes.c_float, _vp, _vp, _DESC, _vp]
lib.pa_append_kv_e4m3.restype = ctypes.c_int
lib.pa_copy_blocks.restype = ctypes.c_int
lib.pa_pool_create.argtypes = [_i32, _vp, _i32, ctypes.POINTER(_vp)]
lib.pa_pool_create.restype = ctypes.c_int
lib.pa_pool_destroy.argtypes = [_vp]
lib.pa_pool_destroy.restype = None
lib.pa_pool_alloc.argtypes = [_vp, _i32, _vp]
lib.pa_pool_alloc.restype = ctypes.c_int
lib.pa_pool_share.argtypes = [_vp, _i32]
lib.pa_pool_share.restype = ctypes.c_int
lib.pa_pool_free.argtypes = [_vp, _i32]
lib.pa_pool_free.restype = ctypes.c_int
lib.pa_pool_num_free.argtypes = [_vp]
lib.pa_pool_num_free.restype = _i32
lib.pa_pool_refcount.argtypes = [_vp, _i32]
lib.pa_pool_refcount.restype = _i32


def pa_status_string(status: int) -> str:
    return lib.pa_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


def declared_symbols(header: str = HEADER) -> list:
    """Function names include/pa.h declares (used by the ABI tests)."""
    text = open(header).read()
    return sorted(set(re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, re.M)))


# ---- pointer marshalling ----------------------------------------------------------------
def _dev(t, dtype_name: str, what: str):
    """Device pointer of a contiguous CUDA tensor of the given torch dtype (or a raw int)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    import torch
    want = getattr(torch, dtype_name)
    if t.dtype != want:
        raise TypeError("%s: expected %s, got %s" % (what, want, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % what)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % what)
    return t.data_ptr()


def _cache(t, desc: "CacheDesc", what: str, options=None):
    """Device pointer of a KV cache tensor (bf16, or uint8 E4M3 codes when the options say so)
    that holds at least the pool desc describes."""
    if t is not None and not isinstance(t, int):
        need = int(desc.num_blocks) * desc.num_kv_heads * desc.block_size * desc.head_dim
        if t.numel() < need:
            raise ValueError("%s holds %d elements, the pool described needs %d" % (what, t.numel(), need))
    e4m3 = options is not None and options.kv_dtype == PA_KV_E4M3
    return _dev(t, "uint8" if e4m3 else "bfloat16", what)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _host(a: np.ndarray, dtype, what: str) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (what, np.dtype(dtype), a.dtype))
    return a


# ---- KV append / decode -----------------------------------------------------------------
def pa_append_kv(k, v, slot_mapping, k_cache, v_cache, desc: CacheDesc, stream=None,
                 num_tokens: int | None = None) -> None:
    n = int(slot_mapping.shape[0]) if num_tokens is None else int(num_tokens)
    _check(lib.pa_append_kv(_dev(k, "bfloat16", "k"), _dev(v, "bfloat16", "v"),
                            _dev(slot_mapping, "int64", "slot_mapping"), n,
                            _cache(k_cache, desc, "k_cache"), _cache(v_cache, desc, "v_cache"),
                            ctypes.byref(desc), _stream(stream)), "pa_append_kv")


def pa_append_kv_e4m3(k, v, slot_mapping, k_scale: float, v_scale: float, k_cache, v_cache,
                      desc: CacheDesc, stream=None, num_tokens: int | None = None) -> None:
    """Quantizing append into uint8 E4M3 pools."""
    n = int(slot_mapping.shape[0]) if num_tokens is None else int(num_tokens)
    e4m3 = DecodeOptions(kv_dtype=PA_KV_E4M3)
    _check(lib.pa_append_kv_e4m3(_dev(k, "bfloat16", "k"), _dev(v, "bfloat16", "v"),
                                 _dev(slot_mapping, "int64", "slot_mapping"), n, float(k_scale),
                                 float(v_scale), _cache(k_cache, desc, "k_cache", e4m3),
                                 _cache(v_cache, desc, "v_cache", e4m3), ctypes.byref(desc),
                                 _stream(stream)), "pa_append_kv_e4m3")


def pa_rope_append_kv(q, q_out, k, v, positions, slot_mapping, rope_theta: float, k_cache, v_cache,
                      desc: CacheDesc, stream=None, num_tokens: int | None = None) -> None:
    n = int(slot_mapping.shape[0]) if num_tokens is None else int(num_tokens)
    _check(lib.pa_rope_append_kv(_dev(q, "bfloat16", "q"), _dev(q_out, "bfloat16", "q_out"),
                                 _dev(k, "bfloat16", "k"), _dev(v, "bfloat16", "v"),
                                 _dev(positions, "int32", "positions"),
                                 _dev(slot_mapping, "int64", "slot_mapping"), n, float(rope_theta),
                                 _cache(k_cache, desc, "k_cache"), _cache(v_cache, desc, "v_cache"),
                                 ctypes.byref(desc), _stream(stream)), "pa_rope_append_kv")


def pa_copy_blocks(k_cache, v_cache, copies, desc: CacheDesc, stream=None) -> None:
    """Device copy-on-write: copies is a device int32 [n, 2] tensor of (src, dst) block pairs."""
    n = int(copies.shape[0])
    _check(lib.pa_copy_blocks(_cache(k_cache, desc, "k_cache"), _cache(v_cache, desc, "v_cache"),
                              _dev(copies, "int32", "copies") if n else None, n, ctypes.byref(desc),
                              _stream(stream)), "pa_copy_blocks")


PA_PREFILL_AUTO, PA_PREFILL_TCGEN05, PA_PREFILL_MMA, PA_PREFILL_TCGEN05_WS = 0, 1, 2, 3
_PREFILL_KERNELS = {"auto": PA_PREFILL_AUTO, "tcgen05": PA_PREFILL_TCGEN05, "mma": PA_PREFILL_MMA,
                    "tcgen05_ws": PA_PREFILL_TCGEN05_WS}


def pa_prefill(q, k_cache, v_cache, block_tables, cu_seqlens_q, context_lens, max_q_len: int, scale: float,
               out, workspace, desc: CacheDesc, stream=None, kernel: str = "auto") -> None:
    """Causal attention of each sequence's last Tq tokens over its paged cache.

    kernel: "auto" ("tcgen05_ws" where it serves the block size, else "tcgen05"), "tcgen05",
    "tcgen05_ws" or "mma" (the warp-level mma.sync kernel)."""
    n = int(context_lens.shape[0])
    if kernel not in _PREFILL_KERNELS:
        raise ValueError("pa_prefill: kernel must be one of %s" % sorted(_PREFILL_KERNELS))
    _check(lib.pa_prefill(_dev(q, "bfloat16", "q"), _cache(k_cache, desc, "k_cache"),
                          _cache(v_cache, desc, "v_cache"), _dev(block_tables, "int32", "block_tables"),
                          _dev(cu_seqlens_q, "int32", "cu_seqlens_q"), _dev(context_lens, "int32", "context_lens"),
                          n, int(max_q_len), float(scale), _dev(out, "bfloat16", "out"),
                          _dev(workspace, "uint8", "workspace"), int(workspace.numel()), ctypes.byref(desc),
                          _PREFILL_KERNELS[kernel], _stream(stream)), "pa_prefill")


def pa_decode_workspace_size(num_seqs: int, max_context_len: int, desc: CacheDesc,
                             options: DecodeOptions | None = None) -> int:
    n = lib.pa_decode_workspace_size_ex(int(num_seqs), int(max_context_len), ctypes.byref(desc),
                                        ctypes.byref(options) if options is not None else None)
    if n == 0:
        raise PaError(-1, "pa_decode_workspace_size")
    return int(n)


def pa_decode_max_splits(num_seqs: int, max_context_len: int, desc: CacheDesc,
                         options: DecodeOptions | None = None) -> int:
    return int(lib.pa_decode_max_splits(int(num_seqs), int(max_context_len), ctypes.byref(desc),
                                        ctypes.byref(options) if options is not None else None))


def pa_decode_describe(num_seqs: int, max_context_len: int, desc: CacheDesc,
                       options: DecodeOptions | None = None) -> DecodePlanInfo:
    """The decode kernel and partition a call of this shape runs (kernel, ctas, split_tokens,
    max_splits)."""
    info = DecodePlanInfo()
    _check(lib.pa_decode_describe(int(num_seqs), int(max_context_len), ctypes.byref(desc),
                                  ctypes.byref(options) if options is not None else None,
                                  ctypes.byref(info)), "pa_decode_describe")
    return info


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
              out, workspace, desc: CacheDesc, options: DecodeOptions | None = None, stream=None,
              num_seqs: int | None = None, workspace_bytes: int | None = None) -> None:
    n = int(context_lens.shape[0]) if num_seqs is None else int(num_seqs)
    wbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else int(workspace_bytes)
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    _check(lib.pa_decode_ex(_dev(q, "bfloat16", "q"), _cache(k_cache, desc, "k_cache", options),
                            _cache(v_cache, desc, "v_cache", options),
                            _dev(block_tables, "int32", "block_tables"),
                            _dev(context_lens, "int32", "context_lens"), n, int(max_context_len),
                            float(scale), _dev(out, "bfloat16", "out"), ws, wbytes,
                            ctypes.byref(desc),
                            ctypes.byref(options) if options is not None else None,
                            _stream(stream)), "pa_decode")


def pa_append_decode(q, k, v, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                     scale: float, out, workspace, desc: CacheDesc,
                     options: DecodeOptions | None = None, stream=None, num_seqs: int | None = None,
                     workspace_bytes: int | None = None) -> None:
    """Append each sequence's newest token at position context_lens-1, then decode."""
    n = int(context_lens.shape[0]) if num_seqs is None else int(num_seqs)
    wbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else int(workspace_bytes)
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    _check(lib.pa_append_decode(_dev(q, "bfloat16", "q"), _dev(k, "bfloat16", "k"),
                                _dev(v, "bfloat16", "v"), _cache(k_cache, desc, "k_cache", options),
                                _cache(v_cache, desc, "v_cache", options),
                                _dev(block_tables, "int32", "block_tables"),
                                _dev(context_lens, "int32", "context_lens"), n,
                                int(max_context_len), float(scale), _dev(out, "bfloat16", "out"), ws,
                                wbytes, ctypes.byref(desc),
                                ctypes.byref(options) if options is not None else None,
                                _stream(stream)), "pa_append_decode")


def pa_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                      scale: float, out, desc: CacheDesc, options: DecodeOptions | None = None,
                      stream=None, num_seqs: int | None = None) -> None:
    """pa_decode with the library's fixed scratch array instead of a caller workspace."""
    n = int(context_lens.shape[0]) if num_seqs is None else int(num_seqs)
    _check(lib.pa_decode_noalloc(_dev(q, "bfloat16", "q"), _cache(k_cache, desc, "k_cache", options),
                                 _cache(v_cache, desc, "v_cache", options),
                                 _dev(block_tables, "int32", "block_tables"),
                                 _dev(context_lens, "int32", "context_lens"), n,
                                 int(max_context_len), float(scale), _dev(out, "bfloat16", "out"),
                                 ctypes.byref(desc),
                                 ctypes.byref(options) if options is not None else None,
                                 _stream(stream)), "pa_decode_noalloc")


def pa_decode_status(workspace, stream=None, workspace_bytes: int | None = None) -> int:
    wbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else int(workspace_bytes)
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    return int(lib.pa_decode_status(ws, wbytes, _stream(stream)))


def pa_slot_mapping(block_tables: np.ndarray, lengths: np.ndarray, block_size: int) -> np.ndarray:
    bt = _host(block_tables, np.int32, "block_tables")
    ln = _host(lengths, np.int32, "lengths")
    out = np.empty(ln.shape[0], dtype=np.int64)
    _check(lib.pa_slot_mapping(bt.ctypes.data, bt.shape[1], ln.ctypes.data, ln.shape[0],
                               int(block_size), out.ctypes.data), "pa_slot_mapping")
    return out


# ---- host block manager -----------------------------------------------------------------
class BlockManager:
    """Owner of a pa_block_manager handle (host memory only)."""

    def __init__(self, num_blocks: int, block_size: int, max_seqs: int, max_blocks_per_seq: int,
                 free_order):
        fo = _host(np.asarray(free_order, dtype=np.int32), np.int32, "free_order")
        h = _vp()
        _check(lib.pa_bm_create(int(num_blocks), int(block_size), int(max_seqs),
                                int(max_blocks_per_seq), fo.ctypes.data if fo.size else None,
                                int(fo.size), ctypes.byref(h)), "pa_bm_create")
        self._h = h
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self.max_seqs, self.max_blocks_per_seq = int(max_seqs), int(max_blocks_per_seq)

    def close(self):
        if getattr(self, "_h", None):
            lib.pa_bm_destroy(self._h)
            self._h = None

    __del__ = close

    def import_seq(self, seq: int, num_tokens: int, blocks) -> None:
        b = _host(np.asarray(blocks, dtype=np.int32), np.int32, "blocks")
        _check(lib.pa_bm_import_seq(self._h, int(seq), int(num_tokens),
                                    b.ctypes.data if b.size else None), "pa_bm_import_seq")

    def add_seq(self, seq: int, num_tokens: int) -> None:
        _check(lib.pa_bm_add_seq(self._h, int(seq), int(num_tokens)), "pa_bm_add_seq")

    def fork_seq(self, seq: int, src: int, num_shared_blocks: int, num_tokens: int) -> None:
        _check(lib.pa_bm_fork_seq(self._h, int(seq), int(src), int(num_shared_blocks),
                                  int(num_tokens)), "pa_bm_fork_seq")

    def free_seq(self, seq: int) -> None:
        _check(lib.pa_bm_free_seq(self._h, int(seq)), "pa_bm_free_seq")

    def append_tokens(self, seqs, out: np.ndarray | None = None) -> np.ndarray:
        s = _host(np.asarray(seqs, dtype=np.int32), np.int32, "seqs")
        slots = out if out is not None else np.empty(s.size, dtype=np.int64)
        _check(lib.pa_bm_append_tokens(self._h, s.ctypes.data, int(s.size), slots.ctypes.data),
               "pa_bm_append_tokens")
        return slots

    def add_seq_tokens(self, seq: int, token_ids) -> int:
        """Admit by token ids (prefix caching); returns the number of tokens found cached."""
        t = _host(np.asarray(token_ids, dtype=np.int32), np.int32, "token_ids")
        cached = ctypes.c_int32(0)
        _check(lib.pa_bm_add_seq_tokens(self._h, int(seq), t.ctypes.data if t.size else None,
                                        int(t.size), ctypes.byref(cached)), "pa_bm_add_seq_tokens")
        return int(cached.value)

    def fork_all(self, seq: int, src: int) -> None:
        _check(lib.pa_bm_fork_all(self._h, int(seq), int(src)), "pa_bm_fork_all")

    def append_token_ids(self, seqs, token_ids):
        """Appends with ids and copy-on-write; returns (slots int64 [n], copies int32 [k, 2])."""
        s = _host(np.asarray(seqs, dtype=np.int32), np.int32, "seqs")
        t = _host(np.asarray(token_ids, dtype=np.int32), np.int32, "token_ids")
        if s.size != t.size:
            raise ValueError("seqs and token_ids differ in length")
        slots = np.empty(s.size, dtype=np.int64)
        copies = np.empty((max(s.size, 1), 2), dtype=np.int32)
        nc = ctypes.c_int32(0)
        _check(lib.pa_bm_append_token_ids(self._h, s.ctypes.data, t.ctypes.data, int(s.size),
                                          slots.ctypes.data, copies.ctypes.data, ctypes.byref(nc)),
               "pa_bm_append_token_ids")
        return slots, copies[:nc.value].copy()

    def num_cached_blocks(self) -> int:
        return int(lib.pa_bm_num_cached_blocks(self._h))

    def num_free(self) -> int:
        return int(lib.pa_bm_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(lib.pa_bm_refcount(self._h, int(block)))

    def block_tables(self) -> np.ndarray:
        """Zero-copy numpy view of the manager's [max_seqs, MB] table."""
        p = lib.pa_bm_block_tables(self._h)
        return np.ctypeslib.as_array(p, shape=(self.max_seqs, self.max_blocks_per_seq))

    def context_lens(self) -> np.ndarray:
        p = lib.pa_bm_context_lens(self._h)
        return np.ctypeslib.as_array(p, shape=(self.max_seqs,))

    def take_dirty_rows(self) -> np.ndarray:
        rows = np.empty(self.max_seqs, dtype=np.int32)
        n = lib.pa_bm_take_dirty_rows(self._h, rows.ctypes.data, self.max_seqs)
        return rows[:n]


class BlockPool:
    """Owner of a pa_block_pool handle: per-block alloc / share / free (host memory only)."""

    def __init__(self, num_blocks: int, free_order=None):
        fo = _host(np.asarray(range(num_blocks) if free_order is None else free_order, dtype=np.int32),
                   np.int32, "free_order")
        h = _vp()
        _check(lib.pa_pool_create(int(num_blocks), fo.ctypes.data if fo.size else None, int(fo.size),
                                  ctypes.byref(h)), "pa_pool_create")
        self._h = h
        self.num_blocks = int(num_blocks)

    def close(self):
        if getattr(self, "_h", None):
            lib.pa_pool_destroy(self._h)
            self._h = None

    __del__ = close

    def alloc(self, n: int) -> np.ndarray:
        out = np.empty(max(int(n), 1), dtype=np.int32)
        _check(lib.pa_pool_alloc(self._h, int(n), out.ctypes.data), "pa_pool_alloc")
        return out[:int(n)]

    def share(self, block: int) -> None:
        _check(lib.pa_pool_share(self._h, int(block)), "pa_pool_share")

    def free(self, block: int) -> None:
        _check(lib.pa_pool_free(self._h, int(block)), "pa_pool_free")

    def num_free(self) -> int:
        return int(lib.pa_pool_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(lib.pa_pool_refcount(self._h, int(block)))
