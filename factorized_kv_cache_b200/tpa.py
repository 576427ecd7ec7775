"""Python binding of libtpa (include/tpa.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors are
PyTorch CUDA tensors used as plain device buffers; every step of the attention
path runs in the library's CUDA kernels.  There is no fallback: if
``libtpa.so`` is missing, loading raises ``TpaError``.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtpa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "tpa.h")

TPA_OK = 0
TPA_F32, TPA_BF16 = 0, 1
TPA_KERNEL_AUTO, TPA_KERNEL_SIMT, TPA_KERNEL_TENSOR, TPA_KERNEL_TENSOR_SYNC = 0, 1, 2, 3
TPA_DEVERR_APPEND_OVERFLOW = 0x1
TPA_DEVERR_LEN_RANGE = 0x2
TPA_DEVERR_PREFILL_LEN = 0x4
TPA_DEVERR_TIMEOUT = 0x8

STATUS_NAMES = {
    0: "TPA_OK", 1: "TPA_ERR_NULL", 2: "TPA_ERR_SHAPE", 3: "TPA_ERR_UNSUPPORTED",
    4: "TPA_ERR_CAPACITY", 5: "TPA_ERR_WORKSPACE", 6: "TPA_ERR_ALIGNMENT", 7: "TPA_ERR_CUDA",
}

_DTYPES = {TPA_F32: torch.float32, TPA_BF16: torch.bfloat16}


class TpaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class tpa_cache(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("r_k", ctypes.c_int32),
        ("r_v", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("a_k", ctypes.c_void_p),
        ("b_k", ctypes.c_void_p),
        ("a_v", ctypes.c_void_p),
        ("b_v", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
    ]


class tpa_step_plan(ctypes.Structure):
    """Caller-owned storage of a bound decode step (contents private to libtpa)."""
    _fields_ = [("opaque", ctypes.c_uint64 * 256)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtpa.so once and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise TpaError(7, f"{path} is not built; run `python -m factorized_kv_cache_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I32 = ctypes.c_int32
    C = ctypes.POINTER(tpa_cache)
    sig = {
        "tpa_factor_elements_per_token": (ctypes.c_size_t, [I32, I32, I32, I32]),
        "tpa_cache_append": (ctypes.c_int, [C, I32, P, P, P, P, P, P]),
        "tpa_cache_write_slots": (ctypes.c_int, [C, I32, P, P, P, P, P, P, P]),
        "tpa_decode_default_splits": (I32, [C, I32, I32]),
        "tpa_decode_workspace_size": (ctypes.c_size_t, [C, I32, I32, I32]),
        "tpa_decode_attention": (ctypes.c_int, [C, P, P, ctypes.c_float, P, I32, I32, I32, P, ctypes.c_size_t, P]),
        "tpa_decode_attention_noalloc": (ctypes.c_int, [C, P, P, ctypes.c_float, P, I32, I32, I32, P]),
        "tpa_decode_attention_factored": (ctypes.c_int, [C, I32, P, P, P, ctypes.c_float, P, I32, I32, I32, P,
                                                          ctypes.c_size_t, P]),
        "tpa_decode_attention_lse": (ctypes.c_int, [C, P, P, ctypes.c_float, P, P, I32, I32, I32, P, ctypes.c_size_t,
                                                     P]),
        "tpa_merge_lse": (ctypes.c_int, [I32, I32, I32, P, P, P, P, P]),
        "tpa_decode_step": (ctypes.c_int, [C, P, P, P, P, P, I32, P, P, ctypes.c_float, P, I32, I32, I32, I32, P,
                                            ctypes.c_size_t, P]),
        "tpa_stage_async": (ctypes.c_int, [P, P, ctypes.c_size_t, P]),
        "tpa_step_plan_init": (ctypes.c_int, [ctypes.POINTER(tpa_step_plan), C, P, P, P, P, P, I32, P, P,
                                               ctypes.c_float, P, I32, I32, I32, I32, P, ctypes.c_size_t, P, P,
                                               ctypes.c_size_t]),
        "tpa_step_plan_run": (ctypes.c_int, [ctypes.POINTER(tpa_step_plan), P]),
        "tpa_prefill_workspace_size": (ctypes.c_size_t, [C, I32, I32, I32]),
        "tpa_prefill_attention": (ctypes.c_int, [C, I32, I32, P, P, P, ctypes.c_float, P, I32, P, ctypes.c_size_t, P]),
        "tpa_read_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), P]),
        "tpa_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, P]),
        "tpa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "tpa_last_error_message": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def declared_functions(header: str = HEADER_PATH) -> list[str]:
    """Names of the functions include/tpa.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tpa_[a-z0-9_]+)\s*\(", text)))


def _check(status: int):
    if status != TPA_OK:
        msg = load_library().tpa_last_error_message().decode()
        raise TpaError(status, msg)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None) -> ctypes.c_void_p:
    """The cudaStream_t to launch on: `stream`, else the current stream of `device`."""
    if stream is None:
        if _raw_current_stream is not None:
            idx = device.index if device is not None and device.index is not None else torch.cuda.current_device()
            return ctypes.c_void_p(_raw_current_stream(idx))
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


@dataclass
class TpaCache:
    """A factorized KV cache whose planes are caller-owned CUDA tensors."""

    a_k: torch.Tensor      # [B, cap, r_k, h]
    b_k: torch.Tensor      # [B, cap, r_k, d_h], rotated at each token's position
    a_v: torch.Tensor      # [B, cap, r_v, h]
    b_v: torch.Tensor      # [B, cap, r_v, d_h]
    seq_lens: torch.Tensor  # [B] int32
    rope_base: float = 10000.0

    @classmethod
    def allocate(cls, batch, capacity, heads, head_dim, r_k, r_v, dtype=torch.bfloat16,
                 rope_base=10000.0, device="cuda", fill=None):
        kw = dict(dtype=dtype, device=device)
        mk = (lambda *s: torch.full(s, fill, **kw)) if fill is not None else (lambda *s: torch.empty(s, **kw))
        return cls(mk(batch, capacity, r_k, heads), mk(batch, capacity, r_k, head_dim),
                   mk(batch, capacity, r_v, heads), mk(batch, capacity, r_v, head_dim),
                   torch.zeros(batch, dtype=torch.int32, device=device), rope_base)

    @property
    def batch(self):
        return self.a_k.shape[0]

    @property
    def capacity(self):
        return self.a_k.shape[1]

    @property
    def heads(self):
        return self.a_k.shape[3]

    @property
    def head_dim(self):
        return self.b_k.shape[3]

    @property
    def r_k(self):
        return self.a_k.shape[2]

    @property
    def r_v(self):
        return self.a_v.shape[2]

    @property
    def dtype(self):
        return self.a_k.dtype

    def struct(self) -> tpa_cache:
        """The C descriptor, rebuilt (and re-checked) only when a plane tensor or the base changed."""
        planes = (self.a_k, self.b_k, self.a_v, self.b_v, self.seq_lens)
        key = tuple((id(t), t.data_ptr(), t.shape) for t in planes) + (self.rope_base,)
        hit = self.__dict__.get("_struct_cache")
        if hit is not None and hit[0] == key:
            return hit[1]
        s = self._build_struct()
        self.__dict__["_struct_cache"] = (key, s)
        return s

    def _build_struct(self) -> tpa_cache:
        B, cap, rk, h = self.a_k.shape
        d = self.b_k.shape[3]
        rv = self.a_v.shape[2]
        dev = self.a_k.device
        _need(self.a_k, "a_k")
        _need(self.b_k, "b_k", self.a_k.dtype, (B, cap, rk, d), dev)
        _need(self.a_v, "a_v", self.a_k.dtype, (B, cap, rv, h), dev)
        _need(self.b_v, "b_v", self.a_k.dtype, (B, cap, rv, d), dev)
        _need(self.seq_lens, "seq_lens", torch.int32, (B,), dev)
        dt = {torch.float32: TPA_F32, torch.bfloat16: TPA_BF16}.get(self.a_k.dtype)
        if dt is None:
            raise TypeError(f"cache dtype {self.a_k.dtype} is not float32 or bfloat16")
        return tpa_cache(B, cap, h, d, rk, rv, dt, 0, float(self.rope_base),
                         self.a_k.data_ptr(), self.b_k.data_ptr(), self.a_v.data_ptr(), self.b_v.data_ptr(),
                         self.seq_lens.data_ptr())


def tpa_factor_elements_per_token(heads: int, head_dim: int, r_k: int, r_v: int) -> int:
    return int(load_library().tpa_factor_elements_per_token(heads, head_dim, r_k, r_v))


def tpa_status_string(status: int) -> str:
    return load_library().tpa_status_string(status).decode()


def tpa_cache_append(cache: TpaCache, positions, a_k, b_k, a_v, b_v, stream=None):
    """Append n_new tokens per sequence (inputs [B, n_new, R, h|d_h], B_K unrotated)."""
    lib = load_library()
    B = cache.batch
    n_new = positions.shape[1]
    dev, dt = cache.a_k.device, cache.dtype
    _need(positions, "positions", torch.int32, (B, n_new), dev)
    _need(a_k, "a_k", dt, (B, n_new, cache.r_k, cache.heads), dev)
    _need(b_k, "b_k", dt, (B, n_new, cache.r_k, cache.head_dim), dev)
    _need(a_v, "a_v", dt, (B, n_new, cache.r_v, cache.heads), dev)
    _need(b_v, "b_v", dt, (B, n_new, cache.r_v, cache.head_dim), dev)
    s = cache.struct()
    _check(lib.tpa_cache_append(ctypes.byref(s), n_new, _ptr(positions), _ptr(a_k), _ptr(b_k), _ptr(a_v),
                                _ptr(b_v), _stream(stream, dev)))


def tpa_cache_write_slots(cache: TpaCache, slots, positions, a_k, b_k, a_v, b_v, stream=None):
    """Write n_new tokens per sequence at explicit slots [B, n_new]; lengths unchanged."""
    lib = load_library()
    B = cache.batch
    n_new = positions.shape[1]
    dev, dt = cache.a_k.device, cache.dtype
    _need(slots, "slots", torch.int32, (B, n_new), dev)
    _need(positions, "positions", torch.int32, (B, n_new), dev)
    _need(a_k, "a_k", dt, (B, n_new, cache.r_k, cache.heads), dev)
    _need(b_k, "b_k", dt, (B, n_new, cache.r_k, cache.head_dim), dev)
    _need(a_v, "a_v", dt, (B, n_new, cache.r_v, cache.heads), dev)
    _need(b_v, "b_v", dt, (B, n_new, cache.r_v, cache.head_dim), dev)
    s = cache.struct()
    _check(lib.tpa_cache_write_slots(ctypes.byref(s), n_new, _ptr(slots), _ptr(positions), _ptr(a_k), _ptr(b_k),
                                     _ptr(a_v), _ptr(b_v), _stream(stream, dev)))


def tpa_decode_default_splits(cache: TpaCache, max_len: int, kernel: int = TPA_KERNEL_AUTO) -> int:
    s = cache.struct()
    return int(load_library().tpa_decode_default_splits(ctypes.byref(s), max_len, kernel))


def tpa_decode_workspace_size(cache: TpaCache, max_len: int, num_splits: int = 0,
                              kernel: int = TPA_KERNEL_AUTO) -> int:
    s = cache.struct()
    return int(load_library().tpa_decode_workspace_size(ctypes.byref(s), max_len, num_splits, kernel))


def workspace(nbytes: int, device) -> torch.Tensor | None:
    """A 256-byte aligned device buffer of at least nbytes (None for 0)."""
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def tpa_decode_attention(cache: TpaCache, q, q_pos, scale: float | None = None, out=None, max_len: int | None = None,
                         num_splits: int = 0, kernel: int = TPA_KERNEL_AUTO, workspace_buf=None, stream=None):
    """Decode attention; returns out [B, h, d_h] float32."""
    lib = load_library()
    B, h, d = cache.batch, cache.heads, cache.head_dim
    dev = cache.a_k.device
    _need(q, "q", cache.dtype, (B, h, d), dev)
    _need(q_pos, "q_pos", torch.int32, (B,), dev)
    if out is None:
        out = torch.empty(B, h, d, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, (B, h, d), dev)
    if max_len is None:
        max_len = cache.capacity
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    need = int(lib.tpa_decode_workspace_size(ctypes.byref(s), max_len, num_splits, kernel))
    if workspace_buf is None:
        workspace_buf = workspace(need, dev)
    nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
    _check(lib.tpa_decode_attention(ctypes.byref(s), _ptr(q), _ptr(q_pos), float(scale), _ptr(out), max_len,
                                    num_splits, kernel, _ptr(workspace_buf), nbytes, _stream(stream, dev)))
    return out


def tpa_decode_attention_factored(cache: TpaCache, a_q, b_q, q_pos, scale: float | None = None, out=None,
                                  max_len: int | None = None, num_splits: int = 0, kernel: int = TPA_KERNEL_AUTO,
                                  workspace_buf=None, stream=None):
    """Decode attention with the query in TPA form: a_q [B, R_Q, h], b_q [B, R_Q, d_h] (unrotated);
    returns out [B, h, d_h] float32."""
    lib = load_library()
    B, h, d = cache.batch, cache.heads, cache.head_dim
    dev = cache.a_k.device
    r_q = a_q.shape[1]
    _need(a_q, "a_q", cache.dtype, (B, r_q, h), dev)
    _need(b_q, "b_q", cache.dtype, (B, r_q, d), dev)
    _need(q_pos, "q_pos", torch.int32, (B,), dev)
    if out is None:
        out = torch.empty(B, h, d, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, (B, h, d), dev)
    if max_len is None:
        max_len = cache.capacity
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    need = int(lib.tpa_decode_workspace_size(ctypes.byref(s), max_len, num_splits, kernel))
    if workspace_buf is None:
        workspace_buf = workspace(need, dev)
    nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
    _check(lib.tpa_decode_attention_factored(ctypes.byref(s), r_q, _ptr(a_q), _ptr(b_q), _ptr(q_pos), float(scale),
                                             _ptr(out), max_len, num_splits, kernel, _ptr(workspace_buf), nbytes,
                                             _stream(stream, dev)))
    return out


def tpa_decode_step(cache: TpaCache, positions, a_k, b_k, a_v, b_v, q=None, a_q=None, b_q=None,
                    scale: float | None = None, out=None, max_len: int | None = None, advance: bool = True,
                    num_splits: int = 0, kernel: int = TPA_KERNEL_AUTO, workspace_buf=None, stream=None):
    """One fused generation step: store the token's factors (a_k [B, R_K, h], b_k [B, R_K, d_h]
    unrotated, a_v, b_v) at slot seq_lens[b] and attend with its query, dense (q [B, h, d_h]) or
    in TPA form (a_q [B, R_Q, h], b_q [B, R_Q, d_h]), at positions [B]; returns out [B, h, d_h]
    float32.  advance=False leaves seq_lens unchanged."""
    lib = load_library()
    B, h, d = cache.batch, cache.heads, cache.head_dim
    dev, dt = cache.a_k.device, cache.dtype
    _need(positions, "positions", torch.int32, (B,), dev)
    _need(a_k, "a_k", dt, (B, cache.r_k, h), dev)
    _need(b_k, "b_k", dt, (B, cache.r_k, d), dev)
    _need(a_v, "a_v", dt, (B, cache.r_v, h), dev)
    _need(b_v, "b_v", dt, (B, cache.r_v, d), dev)
    if q is not None:
        if a_q is not None or b_q is not None:
            raise ValueError("pass either q or (a_q, b_q)")
        _need(q, "q", dt, (B, h, d), dev)
        r_q, qa, qb = 0, None, q
    else:
        if a_q is None or b_q is None:
            raise ValueError("pass q or both a_q and b_q")
        r_q = a_q.shape[1]
        _need(a_q, "a_q", dt, (B, r_q, h), dev)
        _need(b_q, "b_q", dt, (B, r_q, d), dev)
        qa, qb = a_q, b_q
    if out is None:
        out = torch.empty(B, h, d, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, (B, h, d), dev)
    if max_len is None:
        max_len = cache.capacity
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    if workspace_buf is None:
        workspace_buf = workspace(int(lib.tpa_decode_workspace_size(ctypes.byref(s), max_len, num_splits, kernel)),
                                  dev)
    nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
    _check(lib.tpa_decode_step(ctypes.byref(s), _ptr(positions), _ptr(a_k), _ptr(b_k), _ptr(a_v), _ptr(b_v), r_q,
                               _ptr(qa), _ptr(qb), float(scale), _ptr(out), max_len, 1 if advance else 0, num_splits,
                               kernel, _ptr(workspace_buf), nbytes, _stream(stream, dev)))
    return out


def tpa_decode_attention_lse(cache: TpaCache, q, q_pos, scale: float | None = None, out=None, lse=None,
                             max_len: int | None = None, num_splits: int = 0, kernel: int = TPA_KERNEL_AUTO,
                             workspace_buf=None, stream=None):
    """Decode attention plus each head's log-sum-exp of the scaled scores; returns (out [B, h, d_h],
    lse [B, h]) float32."""
    lib = load_library()
    B, h, d = cache.batch, cache.heads, cache.head_dim
    dev = cache.a_k.device
    _need(q, "q", cache.dtype, (B, h, d), dev)
    _need(q_pos, "q_pos", torch.int32, (B,), dev)
    if out is None:
        out = torch.empty(B, h, d, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(B, h, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, (B, h, d), dev)
    _need(lse, "lse", torch.float32, (B, h), dev)
    if max_len is None:
        max_len = cache.capacity
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    if workspace_buf is None:
        workspace_buf = workspace(int(lib.tpa_decode_workspace_size(ctypes.byref(s), max_len, num_splits, kernel)),
                                  dev)
    nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
    _check(lib.tpa_decode_attention_lse(ctypes.byref(s), _ptr(q), _ptr(q_pos), float(scale), _ptr(out), _ptr(lse),
                                        max_len, num_splits, kernel, _ptr(workspace_buf), nbytes,
                                        _stream(stream, dev)))
    return out, lse


def tpa_merge_lse(parts_out, parts_lse, out=None, lse_out=None, stream=None):
    """Attention over disjoint token sets from each set's (out, lse): parts_out [n, ..., d_h],
    parts_lse [n, ...] float32 -> (out [..., d_h], lse [...])."""
    lib = load_library()
    n, d = parts_out.shape[0], parts_out.shape[-1]
    lead = tuple(parts_out.shape[1:-1])
    dev = parts_out.device
    _need(parts_out, "parts_out", torch.float32, None, dev)
    _need(parts_lse, "parts_lse", torch.float32, (n,) + lead, dev)
    if out is None:
        out = torch.empty(lead + (d,), dtype=torch.float32, device=dev)
    if lse_out is None:
        lse_out = torch.empty(lead, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, lead + (d,), dev)
    _need(lse_out, "lse_out", torch.float32, lead, dev)
    rows = math.prod(lead)
    _check(lib.tpa_merge_lse(n, rows, d, _ptr(parts_out), _ptr(parts_lse), _ptr(out), _ptr(lse_out),
                             _stream(stream, dev)))
    return out, lse_out


def tpa_stage_async(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """Copy ``src`` (pinned host memory) into ``dst`` (device memory, at least as many bytes)
    on ``stream`` (default: the current stream of ``dst``'s device), asynchronously."""
    nbytes = _stage_bytes(dst, src)
    _check(load_library().tpa_stage_async(_ptr(dst), _ptr(src), nbytes, _stream(stream, dst.device)))


def _stage_bytes(dst: torch.Tensor, src: torch.Tensor) -> int:
    if src.device.type != "cpu" or not src.is_pinned():
        raise ValueError("src must be pinned host memory")
    if dst.device.type != "cuda":
        raise ValueError("dst must be device memory")
    if not src.is_contiguous() or not dst.is_contiguous():
        raise ValueError("src and dst must be contiguous")
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError(f"dst holds fewer than the {nbytes} bytes of src")
    return nbytes


class DecodeStepPlan:
    """tpa_decode_step bound to fixed buffers, for a generation loop (tpa_step_plan_init): the
    arguments are checked and marshalled once, and each call is one C call, tpa_step_plan_run,
    with the plan and the stream.  The buffers' contents may change between calls (new factors,
    query, positions); the tensors themselves, and the cache's planes, must stay the same
    objects.  ``out`` may be pinned host memory: the kernels then write the output straight to
    the host.  ``stage=(host_in, dev_in)``: each call first copies ``host_in`` (pinned) into
    ``dev_in`` (the device memory the bound inputs live in) on the same stream, in the same C
    call, for a loop whose inputs come from the host."""

    def __init__(self, cache: TpaCache, positions, a_k, b_k, a_v, b_v, out, q=None, a_q=None, b_q=None,
                 scale: float | None = None, max_len: int | None = None, advance: bool = True, num_splits: int = 0,
                 kernel: int = TPA_KERNEL_AUTO, workspace_buf=None, stage=None):
        lib = load_library()
        B, h, d = cache.batch, cache.heads, cache.head_dim
        dev, dt = cache.a_k.device, cache.dtype
        _need(positions, "positions", torch.int32, (B,), dev)
        _need(a_k, "a_k", dt, (B, cache.r_k, h), dev)
        _need(b_k, "b_k", dt, (B, cache.r_k, d), dev)
        _need(a_v, "a_v", dt, (B, cache.r_v, h), dev)
        _need(b_v, "b_v", dt, (B, cache.r_v, d), dev)
        if out.device.type == "cpu":
            # pinned host memory is addressable by the kernels: the step writes its output there
            # directly, with no separate device-to-host copy
            if not out.is_pinned():
                raise ValueError("out on the host must be pinned memory")
            _need(out, "out", torch.float32, (B, h, d))
        else:
            _need(out, "out", torch.float32, (B, h, d), dev)
        if q is not None:
            if a_q is not None or b_q is not None:
                raise ValueError("pass either q or (a_q, b_q)")
            _need(q, "q", dt, (B, h, d), dev)
            r_q, qa, qb = 0, None, q
        else:
            if a_q is None or b_q is None:
                raise ValueError("pass q or both a_q and b_q")
            r_q = a_q.shape[1]
            _need(a_q, "a_q", dt, (B, r_q, h), dev)
            _need(b_q, "b_q", dt, (B, r_q, d), dev)
            qa, qb = a_q, b_q
        if max_len is None:
            max_len = cache.capacity
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        self._struct = cache.struct()
        if workspace_buf is None:
            workspace_buf = workspace(
                int(lib.tpa_decode_workspace_size(ctypes.byref(self._struct), max_len, num_splits, kernel)), dev)
        nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
        self.out = out
        self._keep = (cache, positions, a_k, b_k, a_v, b_v, qa, qb, out, workspace_buf)
        self._device = dev
        staged = (None, None, 0)
        if stage is not None:
            host_in, dev_in = stage
            if dev_in.device != dev:
                raise ValueError(f"stage: dev_in is on {dev_in.device}, expected {dev}")
            staged = (_ptr(dev_in), _ptr(host_in), _stage_bytes(dev_in, host_in))
            self._keep += (host_in, dev_in)
        self._plan = tpa_step_plan()
        with torch.cuda.device(dev):
            _check(lib.tpa_step_plan_init(ctypes.byref(self._plan), ctypes.byref(self._struct), _ptr(positions),
                                          _ptr(a_k), _ptr(b_k), _ptr(a_v), _ptr(b_v), r_q, _ptr(qa), _ptr(qb),
                                          float(scale), _ptr(out), max_len, 1 if advance else 0, num_splits, kernel,
                                          _ptr(workspace_buf), nbytes, *staged))
        self._plan_ref = ctypes.byref(self._plan)
        self._run = lib.tpa_step_plan_run

    def __call__(self, stream=None):
        _check(self._run(self._plan_ref, _stream(stream, self._device)))
        return self.out

    def graph(self, host_in=None, dev_in=None, host_out=None, stream=None):
        """One whole step as a CUDA graph: the copy of ``host_in`` (pinned host memory) into
        ``dev_in`` (the device memory the bound inputs live in), the step, and the copy of the
        output into ``host_out`` (pinned).  Each ``replay()`` runs all three with the buffers'
        current contents, for one graph launch per step; like any CUDA graph it replays on the
        current stream.  Building the graph runs one step first, outside the capture."""
        stream = torch.cuda.Stream(device=self._device) if stream is None else stream
        g = torch.cuda.CUDAGraph()

        def body():
            if host_in is not None:
                dev_in.copy_(host_in, non_blocking=True)
            self(stream)
            if host_out is not None:
                host_out.copy_(self.out, non_blocking=True)

        with torch.cuda.stream(stream):
            body()               # a first run outside the capture (the library's one-time set-up)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            body()
        return g


def tpa_decode_attention_noalloc(cache: TpaCache, q, q_pos, out, scale: float | None = None,
                                 max_len: int | None = None, num_splits: int = 0, kernel: int = TPA_KERNEL_AUTO,
                                 stream=None):
    """Decode attention that allocates nothing: the split partials go to the
    library's built-in 16 MiB scratch array instead of a workspace.  The
    caller passes every buffer, ``out`` included, so this call makes no
    allocation on the Python side either."""
    lib = load_library()
    B, h, d = cache.batch, cache.heads, cache.head_dim
    dev = cache.a_k.device
    _need(q, "q", cache.dtype, (B, h, d), dev)
    _need(q_pos, "q_pos", torch.int32, (B,), dev)
    _need(out, "out", torch.float32, (B, h, d), dev)
    if max_len is None:
        max_len = cache.capacity
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    _check(lib.tpa_decode_attention_noalloc(ctypes.byref(s), _ptr(q), _ptr(q_pos), float(scale), _ptr(out),
                                            max_len, num_splits, kernel, _stream(stream, dev)))
    return out


def tpa_prefill_workspace_size(cache: TpaCache, n_tokens: int, r_q: int, kernel: int = TPA_KERNEL_AUTO) -> int:
    s = cache.struct()
    return int(load_library().tpa_prefill_workspace_size(ctypes.byref(s), n_tokens, r_q, kernel))


def tpa_prefill_attention(cache: TpaCache, a_q, b_q, q_pos, scale: float | None = None, out=None,
                          kernel: int = TPA_KERNEL_AUTO, workspace_buf=None, stream=None):
    """Causal prefill of the last T cache slots; a_q [B,T,R_Q,h], b_q [B,T,R_Q,d_h] unrotated."""
    lib = load_library()
    B, T, r_q = a_q.shape[0], a_q.shape[1], a_q.shape[2]
    h, d = cache.heads, cache.head_dim
    dev = cache.a_k.device
    _need(a_q, "a_q", cache.dtype, (B, T, r_q, h), dev)
    _need(b_q, "b_q", cache.dtype, (B, T, r_q, d), dev)
    _need(q_pos, "q_pos", torch.int32, (B, T), dev)
    if B != cache.batch:
        raise ValueError("a_q batch differs from the cache batch")
    if out is None:
        out = torch.empty(B, T, h, d, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, (B, T, h, d), dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = cache.struct()
    need = int(lib.tpa_prefill_workspace_size(ctypes.byref(s), T, r_q, kernel))
    if workspace_buf is None:
        workspace_buf = workspace(need, dev)
    nbytes = 0 if workspace_buf is None else workspace_buf.numel() * workspace_buf.element_size()
    _check(lib.tpa_prefill_attention(ctypes.byref(s), T, r_q, _ptr(a_q), _ptr(b_q), _ptr(q_pos), float(scale),
                                     _ptr(out), kernel, _ptr(workspace_buf), nbytes, _stream(stream, dev)))
    return out


def tpa_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test: one CTA waits limit_ns on a barrier nothing completes and
    records TPA_DEVERR_TIMEOUT (read it with tpa_read_device_error)."""
    lib = load_library()
    _check(lib.tpa_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def tpa_read_device_error(stream=None) -> int:
    """Synchronise the stream, return and clear the device error word."""
    lib = load_library()
    v = ctypes.c_uint32(0)
    _check(lib.tpa_read_device_error(ctypes.byref(v), _stream(stream)))
    return int(v.value)
