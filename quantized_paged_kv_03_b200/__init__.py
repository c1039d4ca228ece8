"""Python binding of libkvq: a quantized paged KV cache (append, decode
attention and chunked-prefill attention) written for NVIDIA B200 (sm_100a).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels (``csrc/``, C ABI in ``include/kvq.h``).  PyTorch supplies device
memory and streams.  There is no CPU fallback: if ``libkvq.so`` is missing the
import of the library raises.

Formats (see include/kvq.h for the page citations):
    bf16, fp8_row256, int8_g64, nvfp4_g16, k8v4, mxfp8_g32, fp8_tensor
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

FORMATS = {"bf16": 0, "fp8_row256": 1, "int8_g64": 2, "nvfp4_g16": 3, "k8v4": 4,
           "mxfp8_g32": 5, "fp8_tensor": 6}
FORMAT_NAMES = {v: k for k, v in FORMATS.items()}
FLAG_NO_ROTATE = 1
CODES = {"e4m3": 0, "e2m1": 1, "int8": 2, "fp16": 3, "ue4m3": 4}
STATUS_BAD_SLOT, STATUS_BAD_PAGE, STATUS_WAIT_TIMEOUT = 1, 2, 4
NOALLOC_SCRATCH_BYTES = 8 << 20


class KVQError(RuntimeError):
    pass


class _Desc(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("tensor_scales", ctypes.POINTER(ctypes.c_float))]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvq.so; raises if it has not been built (no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise KVQError(f"libkvq.so not found at {LIB_PATH}; build it with "
                       "`python -m quantized_paged_kv_03_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, u32, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                 ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t)
    D = ctypes.POINTER(_Desc)
    sig = {
        "kvq_token_bytes": (sz, [i32, i32]),
        "kvq_row_bytes": (ctypes.c_int, [i32, i32, i32, P, P]),
        "kvq_cache_bytes": (sz, [D]),
        "kvq_cache_create": (ctypes.c_int, [D, P, sz, ctypes.POINTER(P)]),
        "kvq_cache_destroy": (ctypes.c_int, [P]),
        "kvq_append": (ctypes.c_int, [P, i32, P, P, P, i32, P]),
        "kvq_decode_workspace_bytes": (sz, [P, i32, i32, i32]),
        "kvq_decode_attention": (ctypes.c_int, [P, i32, P, i32, P, i32, P, i32, i32, P, i32, f32,
                                                P, sz, P]),
        "kvq_append_decode": (ctypes.c_int, [P, i32, P, P, P, i32, P, i32, P, i32, i32, P, i32, f32,
                                             P, sz, P]),
        "kvq_decode_attention_noalloc": (ctypes.c_int, [P, i32, P, i32, P, i32, P, i32, i32, P, i32,
                                                        f32, P]),
        "kvq_prefill_attention": (ctypes.c_int, [P, i32, P, i32, P, i32, P, i32, P, i32, P, i32, f32,
                                                 P]),
        "kvq_dequant": (ctypes.c_int, [P, i32, P, i32, P, P, P]),
        "kvq_read_rows": (ctypes.c_int, [P, i32, P, i32, P, P, P, P, P]),
        "kvq_encode": (ctypes.c_int, [i32, P, i64, P, P]),
        "kvq_read_device_status": (ctypes.c_int, [P, i32, ctypes.POINTER(u32), P]),
        "kvq_debug_set_wait_polls": (i64, [i64]),
        "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "kvq_version": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def exported_symbols():
    return ["kvq_token_bytes", "kvq_row_bytes", "kvq_cache_bytes", "kvq_cache_create",
            "kvq_cache_destroy", "kvq_append", "kvq_decode_workspace_bytes",
            "kvq_decode_attention", "kvq_append_decode", "kvq_decode_attention_noalloc",
            "kvq_prefill_attention", "kvq_dequant", "kvq_read_rows", "kvq_encode",
            "kvq_read_device_status", "kvq_debug_set_wait_polls", "kvq_status_string", "kvq_version"]


def set_wait_polls(polls: int) -> int:
    """Test surface: polls of a kernel's bounded pipeline wait before it gives
    up (0: at once; negative: the default).  Returns the previous setting."""
    return int(lib().kvq_debug_set_wait_polls(int(polls)))


def _check(status: int, what: str):
    if status != 0:
        msg = lib().kvq_status_string(status).decode()
        raise KVQError(f"{what}: {msg} (status {status})")


def _fmt(f) -> int:
    return FORMATS[f] if isinstance(f, str) else int(f)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_tensor(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise KVQError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise KVQError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise KVQError(f"{name} must be contiguous")
    return t


def token_bytes(fmt, head_dim: int) -> int:
    """K+V bytes per token per kv-head (codes + scales)."""
    return int(lib().kvq_token_bytes(_fmt(fmt), head_dim))


def row_bytes(fmt, head_dim: int, is_v: bool):
    cb, sb = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().kvq_row_bytes(_fmt(fmt), head_dim, int(is_v), ctypes.byref(cb), ctypes.byref(sb)),
           "row_bytes")
    return cb.value, sb.value


def _desc(fmt, head_dim, n_kv_heads, page_size, num_pages, num_layers, flags, tensor_scales):
    d = _Desc(_fmt(fmt), head_dim, n_kv_heads, page_size, num_pages, num_layers, flags, None)
    keep = None
    if tensor_scales is not None:
        flat = [float(x) for pair in tensor_scales for x in pair]
        keep = (ctypes.c_float * len(flat))(*flat)
        d.tensor_scales = ctypes.cast(keep, ctypes.POINTER(ctypes.c_float))
    return d, keep


def cache_bytes(fmt, head_dim, n_kv_heads, page_size, num_pages, num_layers=1, flags=0) -> int:
    d, _ = _desc(fmt, head_dim, n_kv_heads, page_size, num_pages, num_layers, flags, None)
    return int(lib().kvq_cache_bytes(ctypes.byref(d)))


def encode(code, x, out=None, stream=None):
    """Element-wise encoder of the append kernel (test surface): uint8 codes
    (two bytes per value for fp16)."""
    import torch
    code = CODES[code] if isinstance(code, str) else int(code)
    _dev_tensor(x, torch.float32, "x")
    w = 2 if code == CODES["fp16"] else 1
    if out is None:
        out = torch.empty(x.numel() * w, dtype=torch.uint8, device=x.device)
    _check(lib().kvq_encode(code, _ptr(x), x.numel(), _ptr(out), _stream(stream)), "encode")
    return out


class KVCache:
    """A paged KV cache in one storage format.  The pool is a torch uint8 tensor
    of ``cache_bytes(...)`` bytes on the current CUDA device."""

    def __init__(self, fmt, head_dim: int, n_kv_heads: int, page_size: int, num_pages: int,
                 num_layers: int = 1, flags: int = 0, tensor_scales=None, device=None):
        import torch
        self.format = _fmt(fmt)
        self.head_dim, self.n_kv_heads, self.page_size = head_dim, n_kv_heads, page_size
        self.num_pages, self.num_layers, self.flags = num_pages, num_layers, flags
        d, keep = _desc(fmt, head_dim, n_kv_heads, page_size, num_pages, num_layers, flags,
                        tensor_scales)
        nbytes = int(lib().kvq_cache_bytes(ctypes.byref(d)))
        if nbytes == 0:
            raise KVQError(f"invalid cache descriptor ({FORMAT_NAMES.get(self.format)}, D={head_dim}, "
                           f"H={n_kv_heads}, P={page_size})")
        self.pool = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.pool[:256].zero_()
        h = ctypes.c_void_p()
        _check(lib().kvq_cache_create(ctypes.byref(d), _ptr(self.pool), nbytes, ctypes.byref(h)),
               "cache_create")
        self._h = h
        self._ws = None
        del keep

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.kvq_cache_destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def row_bytes(self, is_v: bool):
        return row_bytes(self.format, self.head_dim, is_v)

    def append(self, layer: int, k, v, slot_mapping, stream=None):
        """k, v: bf16 [T, H_kv, D]; slot_mapping: int64 [T] (negative = skip)."""
        import torch
        _dev_tensor(k, torch.bfloat16, "k")
        _dev_tensor(v, torch.bfloat16, "v")
        _dev_tensor(slot_mapping, torch.int64, "slot_mapping")
        T = slot_mapping.numel()
        if k.numel() != T * self.n_kv_heads * self.head_dim or v.numel() != k.numel():
            raise KVQError("append: k/v must be [T, H_kv, D] matching slot_mapping")
        _check(lib().kvq_append(self._h, layer, _ptr(k), _ptr(v), _ptr(slot_mapping), T,
                                _stream(stream)), "append")

    def decode_workspace_bytes(self, batch: int, n_q_heads: int, max_seq_len: int) -> int:
        return int(lib().kvq_decode_workspace_bytes(self._h, batch, n_q_heads, max_seq_len))

    def workspace(self, batch: int, n_q_heads: int, max_seq_len: int):
        """A zeroed workspace tensor for these sizes (kept and reused while large enough)."""
        import torch
        need = self.decode_workspace_bytes(batch, n_q_heads, max_seq_len)
        if need == 0:
            raise KVQError("decode_workspace_bytes: unsupported sizes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=self.pool.device)
        return self._ws

    def decode_attention(self, layer: int, q, block_table, seq_lens, max_seq_len: int, out=None,
                         out_fp32: bool = True, softmax_scale: float = 0.0, workspace=None,
                         stream=None):
        """q: bf16 [B, Hq, D]; block_table: int32 [B, max_pages]; seq_lens: int32 [B]."""
        import torch
        _dev_tensor(q, torch.bfloat16, "q")
        _dev_tensor(block_table, torch.int32, "block_table")
        _dev_tensor(seq_lens, torch.int32, "seq_lens")
        B, Hq, D = q.shape
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                              device=q.device)
        else:
            _dev_tensor(out, torch.float32 if out_fp32 else torch.bfloat16, "out")
        ws = self.workspace(B, Hq, max_seq_len) if workspace is None else workspace
        _check(lib().kvq_decode_attention(self._h, layer, _ptr(q), Hq, _ptr(block_table),
                                          block_table.shape[1], _ptr(seq_lens), B, max_seq_len,
                                          _ptr(out), int(out_fp32), float(softmax_scale),
                                          _ptr(ws), ws.numel(), _stream(stream)),
               "decode_attention")
        return out

    def append_decode(self, layer: int, k_new, v_new, q, block_table, seq_lens, max_seq_len: int,
                      out=None, out_fp32: bool = True, softmax_scale: float = 0.0, workspace=None,
                      stream=None):
        """One decode step in one launch: append token seq_len[b] - 1 of every
        sequence (k_new, v_new: bf16 [B, H_kv, D]) and attend over [0, seq_len)."""
        import torch
        _dev_tensor(k_new, torch.bfloat16, "k_new")
        _dev_tensor(v_new, torch.bfloat16, "v_new")
        _dev_tensor(q, torch.bfloat16, "q")
        _dev_tensor(block_table, torch.int32, "block_table")
        _dev_tensor(seq_lens, torch.int32, "seq_lens")
        B, Hq, D = q.shape
        if k_new.numel() != B * self.n_kv_heads * D or v_new.numel() != k_new.numel():
            raise KVQError("append_decode: k_new/v_new must be [B, H_kv, D]")
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                              device=q.device)
        else:
            _dev_tensor(out, torch.float32 if out_fp32 else torch.bfloat16, "out")
        ws = self.workspace(B, Hq, max_seq_len) if workspace is None else workspace
        _check(lib().kvq_append_decode(self._h, layer, _ptr(k_new), _ptr(v_new), _ptr(q), Hq,
                                       _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B,
                                       max_seq_len, _ptr(out), int(out_fp32), float(softmax_scale),
                                       _ptr(ws), ws.numel(), _stream(stream)),
               "append_decode")
        return out

    def decode_attention_noalloc(self, layer: int, q, block_table, seq_lens, max_seq_len: int, out,
                                 out_fp32: bool = True, softmax_scale: float = 0.0, stream=None):
        """decode_attention for callers that cannot allocate device memory: the
        scratch lives in a fixed 8 MiB array inside the library, so no workspace
        is passed and nothing is allocated (the caller still provides `out`).
        Calls that overlap on the GPU share that array and must not run
        concurrently; the first call on a device should come before any stream
        capture."""
        import torch
        _dev_tensor(q, torch.bfloat16, "q")
        _dev_tensor(block_table, torch.int32, "block_table")
        _dev_tensor(seq_lens, torch.int32, "seq_lens")
        _dev_tensor(out, torch.float32 if out_fp32 else torch.bfloat16, "out")
        B, Hq, D = q.shape
        _check(lib().kvq_decode_attention_noalloc(self._h, layer, _ptr(q), Hq, _ptr(block_table),
                                                  block_table.shape[1], _ptr(seq_lens), B, max_seq_len,
                                                  _ptr(out), int(out_fp32), float(softmax_scale),
                                                  _stream(stream)),
               "decode_attention_noalloc")
        return out

    def prefill_attention(self, layer: int, q, cu_q_lens, block_table, seq_lens, max_q_len: int | None = None,
                          out=None, out_fp32: bool = True, softmax_scale: float = 0.0, stream=None):
        """Causal attention of a chunk of query tokens per sequence (chunked
        prefill).  q: bf16 [total_q, Hq, D], the rows of sequence b being
        cu_q_lens[b] .. cu_q_lens[b+1]-1 (int32 [B+1]); seq_lens: int32 [B]
        cached tokens, the chunk included (append its K/V first).  Query token
        i of sequence b attends positions [0, seq_lens[b] - n_b + i].
        max_q_len (the longest chunk) sizes the grid; None reads it from
        cu_q_lens (a device-to-host copy)."""
        import torch
        _dev_tensor(q, torch.bfloat16, "q")
        _dev_tensor(cu_q_lens, torch.int32, "cu_q_lens")
        _dev_tensor(block_table, torch.int32, "block_table")
        _dev_tensor(seq_lens, torch.int32, "seq_lens")
        Tq, Hq, D = q.shape
        B = seq_lens.numel()
        if cu_q_lens.numel() != B + 1:
            raise KVQError("prefill_attention: cu_q_lens must hold batch + 1 offsets")
        if max_q_len is None:
            max_q_len = int((cu_q_lens[1:] - cu_q_lens[:-1]).max().item()) if B else 0
        if out is None:
            out = torch.empty((Tq, Hq, D), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                              device=q.device)
        else:
            _dev_tensor(out, torch.float32 if out_fp32 else torch.bfloat16, "out")
        _check(lib().kvq_prefill_attention(self._h, layer, _ptr(q), Hq, _ptr(cu_q_lens), int(max_q_len),
                                           _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B,
                                           _ptr(out), int(out_fp32), float(softmax_scale),
                                           _stream(stream)),
               "prefill_attention")
        return out

    def dequant(self, layer: int, slots, stream=None):
        """fp32 K and V [n, H_kv, D] of the given slots, stored (rotated) domain."""
        import torch
        _dev_tensor(slots, torch.int64, "slots")
        n = slots.numel()
        shape = (n, self.n_kv_heads, self.head_dim)
        k = torch.empty(shape, dtype=torch.float32, device=slots.device)
        v = torch.empty(shape, dtype=torch.float32, device=slots.device)
        _check(lib().kvq_dequant(self._h, layer, _ptr(slots), n, _ptr(k), _ptr(v), _stream(stream)),
               "dequant")
        return k, v

    def read_rows(self, layer: int, slots, stream=None):
        """Logical code and scale bytes of the rows at `slots`:
        (k_codes, k_scales, v_codes, v_scales), uint8 [n, H_kv, bytes]."""
        import torch
        _dev_tensor(slots, torch.int64, "slots")
        n, H = slots.numel(), self.n_kv_heads
        kcb, ksb = self.row_bytes(False)
        vcb, vsb = self.row_bytes(True)
        dev = slots.device
        kc = torch.zeros((n, H, kcb), dtype=torch.uint8, device=dev)
        ks = torch.zeros((n, H, ksb), dtype=torch.uint8, device=dev)
        vc = torch.zeros((n, H, vcb), dtype=torch.uint8, device=dev)
        vs = torch.zeros((n, H, vsb), dtype=torch.uint8, device=dev)
        _check(lib().kvq_read_rows(self._h, layer, _ptr(slots), n, _ptr(kc), _ptr(ks) if ksb else None,
                                   _ptr(vc), _ptr(vs) if vsb else None, _stream(stream)),
               "read_rows")
        return kc, ks, vc, vs

    def read_device_status(self, clear: bool = False, stream=None) -> int:
        st = ctypes.c_uint32()
        _check(lib().kvq_read_device_status(self._h, int(clear), ctypes.byref(st), _stream(stream)),
               "read_device_status")
        return st.value
