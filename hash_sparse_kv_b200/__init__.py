"""Python binding of libhkv (the B200 hash-code KV retrieval library).

Argument marshalling only: every function here checks tensor shapes, dtypes
and devices, then calls the C entry point of the same name in libhkv.so with
raw device pointers and the current CUDA stream.  All work runs in the
library's CUDA kernels.  There is no CPU fallback: if libhkv.so is missing the
import of any entry point raises.

    import hash_sparse_kv_b200 as hkv
    qh = hkv.HashParams.lsh(R)                     # R [bits, 128] on cuda
    hkv.hkv_encode_keys(qh, K.view(-1, 128), codes.view(-1, W))
    ws = hkv.workspace(B, Hq, Hkv, N, bits, top_k, n_sink, n_local)
    hkv.hkv_retrieve_topk(q_codes, k_codes, N, n_sink, n_local, top_k, idx, ws=ws)
    hkv.hkv_sparse_attend(q, K, V, N, idx, n_sink, n_local, out, ws=ws)
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "HKV_OK", "HKV_ERR_INVALID_ARG", "HKV_ERR_UNSUPPORTED", "HKV_ERR_CAPACITY", "HKV_ERR_CUDA",
    "HKV_ERR_TIMEOUT", "HKV_ERR_DEVICE_RANGE", "HKV_F32", "HKV_BF16", "HKV_HASH_LSH", "HKV_HASH_MLP",
    "HKV_HASH_SIGN", "HKV_HASH_NONE", "HkvError", "HashParams", "lib", "lib_path", "workspace", "status_word",
    "hkv_version", "hkv_last_error", "hkv_check", "hkv_workspace_bytes", "hkv_workspace_reset",
    "hkv_encode_keys", "hkv_mlp_pack_bytes", "hkv_mlp_pack", "hkv_append", "hkv_retrieve_topk",
    "hkv_retrieve_topk_static", "hkv_retrieve_topk_heads", "hkv_retrieve_topk_normw", "hkv_sparse_attend",
    "hkv_evict_select", "hkv_write_slots", "hkv_lse_merge", "hkv_decode_step", "hkv_decode_step_heads",
    "hkv_decode_step_ragged", "hkv_split_select", "hkv_lse_merge_n", "hkv_retrieve_topk_paged",
    "hkv_sparse_attend_paged", "hkv_decode_step_paged", "hkv_normw_workspace_bytes", "normw_workspace",
    "hkv_decode_step_normw", "normw_decode_workspace", "hkv_debug_set", "EXPORTS",
]

HKV_OK, HKV_ERR_INVALID_ARG, HKV_ERR_UNSUPPORTED, HKV_ERR_CAPACITY = 0, -1, -2, -3
HKV_ERR_CUDA, HKV_ERR_TIMEOUT, HKV_ERR_DEVICE_RANGE = -4, -5, -6
HKV_F32, HKV_BF16 = 0, 1
HKV_HASH_LSH, HKV_HASH_MLP, HKV_HASH_SIGN, HKV_HASH_NONE = 0, 1, 2, 3

# Every symbol include/hkv.h declares.
EXPORTS = (
    "hkv_last_error", "hkv_version", "hkv_check", "hkv_workspace_bytes", "hkv_workspace_reset",
    "hkv_encode_keys", "hkv_mlp_pack_bytes", "hkv_mlp_pack", "hkv_append", "hkv_retrieve_topk",
    "hkv_retrieve_topk_static", "hkv_retrieve_topk_heads", "hkv_retrieve_topk_normw", "hkv_sparse_attend",
    "hkv_evict_select", "hkv_write_slots", "hkv_lse_merge", "hkv_decode_step", "hkv_decode_step_heads",
    "hkv_decode_step_ragged", "hkv_split_select", "hkv_lse_merge_n", "hkv_retrieve_topk_paged",
    "hkv_sparse_attend_paged", "hkv_decode_step_paged", "hkv_normw_workspace_bytes", "hkv_decode_step_normw",
    "hkv_debug_set",
)

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libhkv.so")


class HkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"hkv error {code}: {msg}")
        self.code = code


class hkv_hash(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("code_bits", ctypes.c_int32),
        ("hidden", ctypes.c_int32), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("R", ctypes.c_void_p), ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
        ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("packed", ctypes.c_void_p),
    ]


_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "hkv_last_error": (ctypes.c_char_p, []),
    "hkv_version": (ctypes.c_char_p, []),
    "hkv_check": (_I, [_P, _P]),
    "hkv_workspace_bytes": (_SZ, [_I, _I, _I, _I64, _I, _I, _I, _I]),
    "hkv_workspace_reset": (_I, [_P, _SZ, _P]),
    "hkv_encode_keys": (_I, [ctypes.POINTER(hkv_hash), _P, _I64, _I64, _P, _I64, _P, _P, _P]),
    "hkv_mlp_pack_bytes": (_SZ, [_I, _I]),
    "hkv_mlp_pack": (_I, [ctypes.POINTER(hkv_hash), _P, _SZ, _P]),
    "hkv_append": (_I, [ctypes.POINTER(hkv_hash), _I, _I, _I, _P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P]),
    "hkv_retrieve_topk": (_I, [_I, _I, _I, _I, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _SZ, _P, _P]),
    "hkv_retrieve_topk_static": (_I, [_I, _I, _I, _I, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _P]),
    "hkv_sparse_attend": (_I, [_I, _I, _I, _I, _P, _P, _P, _I64, _I64, _P, _I, _I, _I, _F, _P, _P, _P, _SZ, _P, _P]),
    "hkv_lse_merge": (_I, [_I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "hkv_decode_step": (_I, [ctypes.POINTER(hkv_hash), _I, _I, _I, _P, _P, _P, _P, _I64, _I64, _I, _I, _I, _F,
                             _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "hkv_debug_set": (_I, [_I, _I64]),
    "hkv_retrieve_topk_heads": (_I, [_I, _I, _I, _I, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _SZ, _P, _P]),
    "hkv_decode_step_heads": (_I, [ctypes.POINTER(hkv_hash), _I, _I, _I, _P, _P, _P, _P, _I64, _I64, _I, _I, _I, _F,
                                   _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "hkv_decode_step_ragged": (_I, [ctypes.POINTER(hkv_hash), _I, _I, _I, _P, _P, _P, _P, _I64, _P, _I64, _I, _I, _I,
                                    _F, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "hkv_retrieve_topk_normw": (_I, [_I, _I, _I, _I, _P, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "hkv_normw_workspace_bytes": (_SZ, [_I, _I, _I64, _I, _I, _I]),
    "hkv_decode_step_normw": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I64, _I64, _I, _I, _I, _F, _P, _P, _P, _P, _P,
                                   _P, _SZ, _P, _P]),
    "hkv_evict_select": (_I, [_I, _I, _I, _I, _P, _P, _I64, _I64, _I, _I, _P, _P, _P, _SZ, _P]),
    "hkv_split_select": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "hkv_lse_merge_n": (_I, [_I, _I64, _P, _P, _P, _P, _P]),
    "hkv_retrieve_topk_paged": (_I, [_I, _I, _I, _I, _P, _P, _P, _I64, _I64, _I, _I64, _I, _I, _I, _P, _P, _P, _SZ, _P,
                                     _P]),
    "hkv_decode_step_paged": (_I, [ctypes.POINTER(hkv_hash), _I, _I, _I, _P, _P, _P, _P, _P, _I64, _I64, _I, _I64, _I,
                                   _I, _I, _F, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "hkv_sparse_attend_paged": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _I64, _I64, _I, _I64, _P, _I, _I, _I, _F, _P, _P,
                                     _P, _SZ, _P, _P]),
    "hkv_write_slots": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P]),
}
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libhkv.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"{lib_path} is missing: build it with `python -m hash_sparse_kv_b200.build`")
        l = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def _ok(rc: int) -> None:
    if rc != HKV_OK:
        raise HkvError(rc, lib().hkv_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HKV_BF16
    if t.dtype == torch.float32:
        return HKV_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str, dtype=None, shape=None, contiguous=True):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_U32 = (torch.int32, torch.uint32) if hasattr(torch, "uint32") else (torch.int32,)


class HashParams:
    """One hash function (the C struct hkv_hash) plus the tensors it points to."""

    def __init__(self, kind: int, dtype: int, code_bits: int, R=None, W1=None, b1=None, W2=None, b2=None):
        self.tensors = [t for t in (R, W1, b1, W2, b2) if t is not None]
        for t in self.tensors:
            _need(t, "hash parameter")
        hidden = 0 if W1 is None else W1.shape[0]
        self.c = hkv_hash(kind, 128, code_bits, hidden, dtype, 0, *(t.data_ptr() if t is not None else None
                                                                      for t in (R, W1, b1, W2, b2)))
        self.kind, self.dtype, self.code_bits = kind, dtype, code_bits

    @property
    def words(self) -> int:
        return self.code_bits // 32

    @classmethod
    def lsh(cls, R: torch.Tensor) -> "HashParams":
        return cls(HKV_HASH_LSH, _dtype_code(R), R.shape[0], R=R)

    @classmethod
    def mlp(cls, W1, b1, W2, b2, dtype: int, pack: bool = True) -> "HashParams":
        """With pack (bf16 inputs only), the 16-bit weight copy that the
        tensor-core encoder reads is written by hkv_mlp_pack on the current stream."""
        for t in (W1, b1, W2, b2):
            _need(t, "MLP weight", torch.float32)
        hp = cls(HKV_HASH_MLP, dtype, W2.shape[0], W1=W1, b1=b1, W2=W2, b2=b2)
        if pack and dtype == HKV_BF16:
            hp.pack()
        return hp

    def pack(self, stream=None) -> None:
        n = lib().hkv_mlp_pack_bytes(self.c.hidden, self.code_bits)
        if n == 0:
            raise ValueError(f"no packed layout for hidden {self.c.hidden}, code_bits {self.code_bits}")
        buf = torch.empty(n, dtype=torch.uint8, device=self.tensors[0].device)
        _ok(lib().hkv_mlp_pack(ctypes.byref(self.c), _ptr(buf), n, _stream(stream)))
        self.packed = buf
        self.c.packed = buf.data_ptr()

    @classmethod
    def sign(cls, dtype: int, head_dim: int = 128) -> "HashParams":
        return cls(HKV_HASH_SIGN, dtype, head_dim)

    @classmethod
    def given(cls, dtype: int, code_bits: int) -> "HashParams":
        """For hkv_decode_step: the query codes are supplied in q_codes."""
        return cls(HKV_HASH_NONE, dtype, code_bits)


def status_word(device=None) -> torch.Tensor:
    """A zeroed int32 device status word."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def hkv_version() -> str:
    return lib().hkv_version().decode()


def hkv_last_error() -> str:
    return lib().hkv_last_error().decode()


def hkv_check(status: torch.Tensor, stream=None) -> int:
    """Synchronize, read and reset the status word; returns its value."""
    return lib().hkv_check(_ptr(status), _stream(stream))


def hkv_debug_set(flags: int, wait_limit_ns: int = 0) -> None:
    _ok(lib().hkv_debug_set(flags, wait_limit_ns))


def hkv_workspace_bytes(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink=0, n_local=0) -> int:
    return lib().hkv_workspace_bytes(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink, n_local)


def hkv_workspace_reset(ws: torch.Tensor, stream=None) -> None:
    _ok(lib().hkv_workspace_reset(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def workspace(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink=0, n_local=0, device=None) -> torch.Tensor:
    """A zero-filled workspace sized by hkv_workspace_bytes."""
    n = hkv_workspace_bytes(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink, n_local)
    if n == 0 and B * Hkv * max(top_k, 1) > 0:
        raise HkvError(HKV_ERR_UNSUPPORTED, hkv_last_error() or "unsupported shape")
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def hkv_encode_keys(h: HashParams, x: torch.Tensor, codes: torch.Tensor, norms: Optional[torch.Tensor] = None,
                    status: Optional[torch.Tensor] = None, stream=None) -> None:
    """x [rows, 128] (row stride may exceed 128) -> codes [rows, code_bits/32]."""
    _need(x, "x", (torch.bfloat16, torch.float32), contiguous=False)
    if x.dim() != 2 or x.shape[1] != 128 or x.stride(1) != 1:
        raise ValueError("x must be [rows, 128] with unit inner stride")
    if _dtype_code(x) != h.dtype:
        raise TypeError("x dtype differs from the hash dtype")
    _need(codes, "codes", _U32, contiguous=False)
    if codes.dim() != 2 or codes.shape[0] != x.shape[0] or codes.shape[1] < h.words or codes.stride(1) != 1:
        raise ValueError("codes must be [rows, >= code_bits/32] with unit inner stride")
    if norms is not None:
        _need(norms, "norms", (torch.float16, torch.int16), shape=(x.shape[0],))
    _ok(lib().hkv_encode_keys(ctypes.byref(h.c), _ptr(x), x.shape[0], x.stride(0), _ptr(codes), codes.stride(0),
                              _ptr(norms), _ptr(status), _stream(stream)))


def hkv_mlp_pack_bytes(hidden: int, code_bits: int) -> int:
    return int(lib().hkv_mlp_pack_bytes(hidden, code_bits))


def hkv_mlp_pack(h: HashParams, packed: torch.Tensor, stream=None) -> None:
    """Writes the 16-bit weight copy of an MLP hash into `packed` (uint8, on the device)."""
    _need(packed, "packed", torch.uint8)
    _ok(lib().hkv_mlp_pack(ctypes.byref(h.c), _ptr(packed), packed.numel(), _stream(stream)))


def hkv_append(h: HashParams, k_new, v_new, K, V, codes, pos: int, norms=None, status=None, stream=None) -> None:
    """k_new, v_new [B, Hkv, T, 128]; K, V [B, Hkv, cap, 128]; codes [B, Hkv, cap, W]."""
    B, Hkv, T, _ = k_new.shape
    cap = K.shape[2]
    _need(k_new, "k_new", shape=(B, Hkv, T, 128))
    _need(v_new, "v_new", shape=(B, Hkv, T, 128))
    _need(K, "K", shape=(B, Hkv, cap, 128))
    _need(V, "V", shape=(B, Hkv, cap, 128))
    _need(codes, "codes", _U32, shape=(B, Hkv, cap, h.words))
    if norms is not None:
        _need(norms, "norms", (torch.float16, torch.int16), shape=(B, Hkv, cap))
    _ok(lib().hkv_append(ctypes.byref(h.c), B, Hkv, T, _ptr(k_new), _ptr(v_new), _ptr(K), _ptr(V), _ptr(codes),
                         _ptr(norms), cap, pos, _ptr(status), _stream(stream)))


def hkv_retrieve_topk(q_codes, k_codes, n_tokens: int, n_sink: int, n_local: int, top_k: int, idx,
                      dist=None, ws=None, status=None, stream=None) -> None:
    """q_codes [B, Hq, W]; k_codes [B, Hkv, cap, W] -> idx [B, Hkv, top_k] (and dist)."""
    B, Hq, W = q_codes.shape
    _, Hkv, cap, W2 = k_codes.shape
    _need(q_codes, "q_codes", _U32)
    _need(k_codes, "k_codes", _U32, shape=(B, Hkv, cap, W))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if dist is not None:
        _need(dist, "dist", torch.int32, shape=(B, Hkv, top_k))
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_retrieve_topk(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(k_codes), cap, n_tokens, n_sink, n_local,
                                top_k, _ptr(idx), _ptr(dist), _ptr(ws), nbytes, _ptr(status), _stream(stream)))


def hkv_retrieve_topk_static(q_codes, k_codes, n_tokens: int, n_sink: int, n_local: int, top_k: int, idx,
                             dist=None, status=None, stream=None) -> None:
    """hkv_retrieve_topk with the library's fixed scratch (no workspace): for
    callers that cannot allocate device memory.  Make the first call on a
    device before any stream capture; calls must not overlap on the GPU."""
    B, Hq, W = q_codes.shape
    _, Hkv, cap, W2 = k_codes.shape
    _need(q_codes, "q_codes", _U32)
    _need(k_codes, "k_codes", _U32, shape=(B, Hkv, cap, W))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if dist is not None:
        _need(dist, "dist", torch.int32, shape=(B, Hkv, top_k))
    _ok(lib().hkv_retrieve_topk_static(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(k_codes), cap, n_tokens, n_sink,
                                       n_local, top_k, _ptr(idx), _ptr(dist), _ptr(status), _stream(stream)))


def hkv_sparse_attend(q, K, V, n_tokens: int, idx, n_sink: int, n_local: int, out, lse=None,
                      scale: Optional[float] = None, ws=None, status=None, stream=None) -> None:
    """q [B, Hq, 128]; K, V [B, Hkv, cap, 128]; idx [B, Hkv, top_k] -> out [B, Hq, 128] fp32."""
    B, Hq, d = q.shape
    _, Hkv, cap, _ = K.shape
    top_k = idx.shape[2]
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(K, "K", q.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", q.dtype, shape=(B, Hkv, cap, d))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_sparse_attend(B, Hq, Hkv, _dtype_code(q), _ptr(q), _ptr(K), _ptr(V), cap, n_tokens, _ptr(idx),
                                top_k, n_sink, n_local, scale, _ptr(out), _ptr(lse), _ptr(ws), nbytes, _ptr(status),
                                _stream(stream)))


def hkv_lse_merge(o1, lse1, o2, lse2, out, lse_out=None, stream=None) -> None:
    """Row-wise log-sum-exp merge of two partial attention results."""
    rows, d = o1.shape
    for t, n in ((o1, "o1"), (o2, "o2"), (out, "out")):
        _need(t, n, torch.float32, shape=(rows, d))
    for t, n in ((lse1, "lse1"), (lse2, "lse2")):
        _need(t, n, torch.float32, shape=(rows,))
    if lse_out is not None:
        _need(lse_out, "lse_out", torch.float32, shape=(rows,))
    _ok(lib().hkv_lse_merge(rows, d, _ptr(o1), _ptr(lse1), _ptr(o2), _ptr(lse2), _ptr(out), _ptr(lse_out),
                            _stream(stream)))


def hkv_retrieve_topk_heads(q_codes, k_codes, n_tokens: int, n_sink: int, n_local: int, top_k: int, idx,
                            dist=None, ws=None, status=None, stream=None) -> None:
    """One index set per query head: idx [B, Hq, top_k] (and dist).  Size ws
    with workspace(B, Hq, Hq, ...)."""
    B, Hq, W = q_codes.shape
    _, Hkv, cap, W2 = k_codes.shape
    _need(q_codes, "q_codes", _U32)
    _need(k_codes, "k_codes", _U32, shape=(B, Hkv, cap, W))
    _need(idx, "idx", torch.int32, shape=(B, Hq, top_k))
    if dist is not None:
        _need(dist, "dist", torch.int32, shape=(B, Hq, top_k))
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_retrieve_topk_heads(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(k_codes), cap, n_tokens, n_sink,
                                      n_local, top_k, _ptr(idx), _ptr(dist), _ptr(ws), nbytes, _ptr(status),
                                      _stream(stream)))


def hkv_decode_step_heads(h: HashParams, q, k_codes, K, V, n_tokens: int, n_sink: int, n_local: int, top_k: int,
                          out, lse=None, q_codes=None, idx=None, scale: Optional[float] = None, ws=None,
                          status=None, stream=None) -> None:
    """hkv_decode_step with one index set per query head (idx [B, Hq, top_k])."""
    B, Hq, d = q.shape
    _, Hkv, cap, W = k_codes.shape
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(k_codes, "k_codes", _U32)
    _need(K, "K", q.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", q.dtype, shape=(B, Hkv, cap, d))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if q_codes is not None:
        _need(q_codes, "q_codes", _U32, shape=(B, Hq, W))
    if idx is not None:
        _need(idx, "idx", torch.int32, shape=(B, Hq, top_k))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_decode_step_heads(ctypes.byref(h.c), B, Hq, Hkv, _ptr(q), _ptr(k_codes), _ptr(K), _ptr(V), cap,
                                    n_tokens, n_sink, n_local, top_k, scale, _ptr(q_codes), _ptr(idx), _ptr(out),
                                    _ptr(lse), _ptr(ws), nbytes, _ptr(status), _stream(stream)))


def hkv_decode_step_ragged(h: HashParams, q, k_codes, K, V, n_tokens_b, n_tokens_max: int, n_sink: int,
                           n_local: int, top_k: int, out, lse=None, q_codes=None, idx=None,
                           scale: Optional[float] = None, ws=None, status=None, stream=None) -> None:
    """hkv_decode_step with per-sequence lengths n_tokens_b (int32 [B], on the device)."""
    B, Hq, d = q.shape
    _, Hkv, cap, W = k_codes.shape
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(k_codes, "k_codes", _U32)
    _need(K, "K", q.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", q.dtype, shape=(B, Hkv, cap, d))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    _need(n_tokens_b, "n_tokens_b", torch.int32, shape=(B,))
    if q_codes is not None:
        _need(q_codes, "q_codes", _U32, shape=(B, Hq, W))
    if idx is not None:
        _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_decode_step_ragged(ctypes.byref(h.c), B, Hq, Hkv, _ptr(q), _ptr(k_codes), _ptr(K), _ptr(V), cap,
                                     _ptr(n_tokens_b), n_tokens_max, n_sink, n_local, top_k, scale, _ptr(q_codes),
                                     _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws), nbytes, _ptr(status),
                                     _stream(stream)))


def hkv_normw_workspace_bytes(B: int, Hkv: int, n_tokens: int, n_sink: int, n_local: int, top_k: int) -> int:
    return lib().hkv_normw_workspace_bytes(B, Hkv, n_tokens, n_sink, n_local, top_k)


def normw_workspace(B, Hkv, n_tokens, n_sink, n_local, top_k, device=None) -> Optional[torch.Tensor]:
    """The workspace of hkv_retrieve_topk_normw for this shape, or None when
    the call runs one block per KV head without one."""
    n = hkv_normw_workspace_bytes(B, Hkv, n_tokens, n_sink, n_local, top_k)
    return None if n == 0 else torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def hkv_retrieve_topk_normw(q_codes, k_codes, norms, n_tokens: int, n_sink: int, n_local: int, top_k: int, idx,
                            score=None, ws=None, stream=None) -> None:
    """Top-k per KV head by the norm-weighted sign score norm * (g * bits - 2 D).
    norms [B, Hkv, cap] fp16 (or its int16 bits); idx [B, Hkv, top_k] int32; score nullable fp32;
    ws nullable (normw_workspace): needed past 65536 candidates per KV head."""
    B, Hq, W = q_codes.shape
    _, Hkv, cap, W2 = k_codes.shape
    _need(q_codes, "q_codes", _U32)
    _need(k_codes, "k_codes", _U32)
    _need(norms, "norms", (torch.float16, torch.int16), shape=(B, Hkv, cap))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if score is not None:
        _need(score, "score", torch.float32, shape=(B, Hkv, top_k))
    if W2 != W:
        raise ValueError("q_codes and k_codes differ in code width")
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_retrieve_topk_normw(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(k_codes), _ptr(norms), cap, n_tokens,
                                      n_sink, n_local, top_k, _ptr(idx), _ptr(score), _ptr(ws), nbytes,
                                      _stream(stream)))


def hkv_split_select(rank: int, Hq: int, code_bits: int, cand_idx, cand_dist, idx, status=None, stream=None) -> None:
    """cand_idx, cand_dist [G, B, Hkv, top_k] int32 (every rank's own top-k, rank-major);
    idx [B, Hkv, top_k] int32 out: rank `rank`'s share of the whole sequence's top-k."""
    G, B, Hkv, k = cand_idx.shape
    _need(cand_idx, "cand_idx", torch.int32)
    _need(cand_dist, "cand_dist", torch.int32, shape=(G, B, Hkv, k))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, k))
    _ok(lib().hkv_split_select(G, rank, B, Hq, Hkv, code_bits, k, _ptr(cand_idx), _ptr(cand_dist), _ptr(idx),
                               _ptr(status), _stream(stream)))


def hkv_lse_merge_n(o, lse, out, lse_out=None, stream=None) -> None:
    """o [G, rows, 128], lse [G, rows] fp32 -> out [rows, 128], lse_out [rows]."""
    G, rows, d = o.shape
    _need(o, "o", torch.float32)
    _need(lse, "lse", torch.float32, shape=(G, rows))
    _need(out, "out", torch.float32, shape=(rows, d))
    if lse_out is not None:
        _need(lse_out, "lse_out", torch.float32, shape=(rows,))
    _ok(lib().hkv_lse_merge_n(G, rows, _ptr(o), _ptr(lse), _ptr(out), _ptr(lse_out), _stream(stream)))


def hkv_retrieve_topk_paged(q_codes, codes_pool, page_table, n_tokens: int, n_sink: int, n_local: int, top_k: int,
                            idx, dist=None, status=None, stream=None, ws=None) -> None:
    """codes_pool [num_pages, Hkv, page_size, W]; page_table [B, max_pages] int32 -> idx [B, Hkv, top_k].
    ws: optional workspace (hkv.workspace of the same shape) for the multi-block path at any length."""
    B, Hq, W = q_codes.shape
    num_pages, Hkv, page_size, W2 = codes_pool.shape
    _need(q_codes, "q_codes", _U32)
    _need(codes_pool, "codes_pool", _U32)
    _need(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if dist is not None:
        _need(dist, "dist", torch.int32, shape=(B, Hkv, top_k))
    if W2 != W:
        raise ValueError("q_codes and codes_pool differ in code width")
    _ok(lib().hkv_retrieve_topk_paged(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(codes_pool), _ptr(page_table),
                                      page_table.shape[1], num_pages, page_size, n_tokens, n_sink, n_local, top_k,
                                      _ptr(idx), _ptr(dist), _ptr(ws),
                                      0 if ws is None else ws.numel() * ws.element_size(), _ptr(status),
                                      _stream(stream)))


def hkv_sparse_attend_paged(q, K_pool, V_pool, page_table, n_tokens: int, idx, n_sink: int, n_local: int, out,
                            lse=None, scale: Optional[float] = None, ws=None, status=None, stream=None) -> None:
    """q [B, Hq, 128]; K_pool, V_pool [num_pages, Hkv, page_size, 128]; page_table [B, max_pages] int32."""
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, _ = K_pool.shape
    top_k = idx.shape[2]
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(K_pool, "K_pool", q.dtype)
    _need(V_pool, "V_pool", q.dtype, shape=tuple(K_pool.shape))
    _need(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_sparse_attend_paged(B, Hq, Hkv, _dtype_code(q), _ptr(q), _ptr(K_pool), _ptr(V_pool),
                                      _ptr(page_table), page_table.shape[1], num_pages, page_size, n_tokens,
                                      _ptr(idx), top_k, n_sink, n_local, scale, _ptr(out), _ptr(lse), _ptr(ws),
                                      nbytes, _ptr(status), _stream(stream)))


def hkv_evict_select(q_codes, k_codes, n_tokens: int, n_sink: int, n_local: int, victim, vdist=None, ws=None,
                     stream=None) -> None:
    """victim [B, Hkv] int32: the most dissimilar non-resident token per KV head."""
    B, Hq, W = q_codes.shape
    _, Hkv, cap, W2 = k_codes.shape
    _need(q_codes, "q_codes", _U32)
    _need(k_codes, "k_codes", _U32)
    _need(victim, "victim", torch.int32, shape=(B, Hkv))
    if vdist is not None:
        _need(vdist, "vdist", torch.int32, shape=(B, Hkv))
    if W2 != W:
        raise ValueError("q_codes and k_codes differ in code width")
    if ws is None:
        ws = torch.zeros(8 * B * Hkv, dtype=torch.uint8, device=q_codes.device)
    _ok(lib().hkv_evict_select(B, Hq, Hkv, W * 32, _ptr(q_codes), _ptr(k_codes), cap, n_tokens, n_sink, n_local,
                               _ptr(victim), _ptr(vdist), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def hkv_write_slots(k_new, v_new, codes_new, K, V, codes, slot, norms_new=None, norms=None, status=None,
                    stream=None) -> None:
    """k_new, v_new [B, Hkv, 128]; codes_new [B, Hkv, W]; slot [B, Hkv] int32 (-1 skips)."""
    B, Hkv, d = k_new.shape
    cap = K.shape[2]
    _need(k_new, "k_new", (torch.bfloat16, torch.float32))
    _need(v_new, "v_new", k_new.dtype, shape=(B, Hkv, d))
    _need(K, "K", k_new.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", k_new.dtype, shape=(B, Hkv, cap, d))
    _need(codes_new, "codes_new", _U32)
    W = codes_new.shape[-1]
    _need(codes, "codes", _U32, shape=(B, Hkv, cap, W))
    _need(slot, "slot", torch.int32, shape=(B, Hkv))
    _ok(lib().hkv_write_slots(B, Hkv, _dtype_code(k_new), W * 32, _ptr(k_new), _ptr(v_new), _ptr(codes_new),
                              _ptr(norms_new), _ptr(K), _ptr(V), _ptr(codes), _ptr(norms), cap, _ptr(slot),
                              _ptr(status), _stream(stream)))


def hkv_decode_step(h: HashParams, q, k_codes, K, V, n_tokens: int, n_sink: int, n_local: int, top_k: int, out,
                    lse=None, q_codes=None, idx=None, scale: Optional[float] = None, ws=None, status=None,
                    stream=None, next_k_codes=None) -> None:
    """One decode step (query encode, retrieval, attention) in the library's kernels.
    next_k_codes: optional hint, the key codes (same shape) the next call will scan."""
    B, Hq, d = q.shape
    _, Hkv, cap, W = k_codes.shape
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(k_codes, "k_codes", _U32)
    _need(K, "K", q.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", q.dtype, shape=(B, Hkv, cap, d))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if q_codes is not None:
        _need(q_codes, "q_codes", _U32, shape=(B, Hq, W))
    if idx is not None:
        _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    if next_k_codes is not None:
        _need(next_k_codes, "next_k_codes", _U32, shape=tuple(k_codes.shape))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_decode_step(ctypes.byref(h.c), B, Hq, Hkv, _ptr(q), _ptr(k_codes), _ptr(K), _ptr(V), cap, n_tokens,
                              n_sink, n_local, top_k, scale, _ptr(q_codes), _ptr(idx), _ptr(out), _ptr(lse),
                              _ptr(next_k_codes), _ptr(ws), nbytes, _ptr(status), _stream(stream)))


def hkv_decode_step_paged(h: HashParams, q, codes_pool, K_pool, V_pool, page_table, n_tokens: int, n_sink: int,
                          n_local: int, top_k: int, out, lse=None, q_codes=None, idx=None, scale: Optional[float] = None,
                          ws=None, status=None, stream=None) -> None:
    """hkv_decode_step over a paged cache: codes_pool [num_pages, Hkv, page_size, W], K_pool and V_pool
    [num_pages, Hkv, page_size, 128], page_table [B, max_pages] int32."""
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, W = codes_pool.shape
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(codes_pool, "codes_pool", _U32)
    _need(K_pool, "K_pool", q.dtype, shape=(num_pages, Hkv, page_size, d))
    _need(V_pool, "V_pool", q.dtype, shape=(num_pages, Hkv, page_size, d))
    _need(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if q_codes is not None:
        _need(q_codes, "q_codes", _U32, shape=(B, Hq, W))
    if idx is not None:
        _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_decode_step_paged(ctypes.byref(h.c), B, Hq, Hkv, _ptr(q), _ptr(codes_pool), _ptr(K_pool),
                                    _ptr(V_pool), _ptr(page_table), page_table.shape[1], num_pages, page_size, n_tokens,
                                    n_sink, n_local, top_k, scale, _ptr(q_codes), _ptr(idx), _ptr(out), _ptr(lse),
                                    _ptr(ws), nbytes, _ptr(status), _stream(stream)))


def normw_decode_workspace(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink=0, n_local=0, device=None) -> torch.Tensor:
    """The workspace of hkv_decode_step_normw's multi-launch step: the segmented retrieval's bytes (rounded up to
    256) then a zero-filled hkv_workspace_bytes workspace."""
    a = hkv_normw_workspace_bytes(B, Hkv, n_tokens, n_sink, n_local, top_k)
    a = (a + 255) // 256 * 256
    n = hkv_workspace_bytes(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink, n_local)
    if n == 0 and B * Hkv * max(top_k, 1) > 0:
        raise HkvError(HKV_ERR_UNSUPPORTED, hkv_last_error() or "unsupported shape")
    return torch.zeros(a + max(n, 256), dtype=torch.uint8, device=device or "cuda")


def hkv_decode_step_normw(q, k_codes, norms, K, V, n_tokens: int, n_sink: int, n_local: int, top_k: int, idx, out,
                          lse=None, score=None, q_codes=None, scale: Optional[float] = None, ws=None, status=None,
                          stream=None) -> None:
    """Norm-weighted sign-VQ decode step: sign query codes, the top_k by norm * (g * bits - 2 D) per KV head,
    attention over the selected, sink and local rows.  q [B, Hq, 128]; k_codes [B, Hkv, cap, W]; norms
    [B, Hkv, cap] fp16; K, V [B, Hkv, cap, 128] in q's dtype; idx [B, Hkv, top_k] int32; out [B, Hq, 128] fp32."""
    B, Hq, d = q.shape
    _, Hkv, cap, W = k_codes.shape
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(k_codes, "k_codes", _U32)
    _need(norms, "norms", (torch.float16, torch.int16), shape=(B, Hkv, cap))
    _need(K, "K", q.dtype, shape=(B, Hkv, cap, d))
    _need(V, "V", q.dtype, shape=(B, Hkv, cap, d))
    _need(idx, "idx", torch.int32, shape=(B, Hkv, top_k))
    _need(out, "out", torch.float32, shape=(B, Hq, d))
    if q_codes is not None:
        _need(q_codes, "q_codes", _U32, shape=(B, Hq, W))
    if score is not None:
        _need(score, "score", torch.float32, shape=(B, Hkv, top_k))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(B, Hq))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _ok(lib().hkv_decode_step_normw(B, Hq, Hkv, _dtype_code(q), W * 32, _ptr(q), _ptr(k_codes), _ptr(norms), _ptr(K),
                                    _ptr(V), cap, n_tokens, n_sink, n_local, top_k, scale, _ptr(q_codes), _ptr(idx),
                                    _ptr(score), _ptr(out), _ptr(lse), _ptr(ws), nbytes, _ptr(status),
                                    _stream(stream)))
