"""Python binding of the iS-KV CUDA library (``libiskv.so``, C ABI in
``include/iskv.h``).

Argument marshalling only: tensors become raw pointers, the current CUDA
stream becomes the ``stream`` argument, status codes become exceptions.
Every step of the method runs in the library's kernels; there is no CPU or
PyTorch fallback, and importing this package fails loudly when the compiled
library is missing (build it with ``python online_rank_kv_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = ["Config", "Cache", "IskvError", "DecodeOperands", "QuantFormat", "quantize_rows",
           "lib_path", "LIB", "F32", "BF16", "WHICH_K", "WHICH_V", "ALL_LAYERS", "FOLD_DEFER_SYNC",
           "EXPORTED"]

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libiskv.so")


if not os.path.exists(lib_path()):
    raise ImportError(
        f"{lib_path()} is missing: build the CUDA library first "
        "(python online_rank_kv_b200/build.py)")

LIB = ctypes.CDLL(lib_path())

OK = 0
F32, BF16 = 0, 1
WHICH_K, WHICH_V = 0, 1
ALL_LAYERS = -1
FOLD_DEFER_SYNC = 1

_ERRORS = {-1: "INVALID_ARG", -2: "CAPACITY", -3: "STATE", -4: "CUDA", -5: "NOCONVERGE",
           -6: "NOMEM", -7: "UNSUPPORTED", -8: "DEVICE_TIMEOUT", -9: "RANGE"}


class IskvError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = _ERRORS.get(code, str(code))
        msg = LIB.iskv_strerror(code).decode()
        super().__init__(f"{where}: ISKV_ERR_{self.name} ({msg})")


class QuantFormat(ctypes.Structure):
    """Mirror of ``iskv_quant_format``: latent-channel code groups."""
    _fields_ = [("groups", ctypes.c_int32), ("channels", ctypes.c_int32 * 4),
                ("bits", ctypes.c_int32 * 4)]

    @classmethod
    def of(cls, groups):
        """From a list of (channels, bits) pairs, first latent channel first."""
        q = cls()
        q.groups = len(groups)
        for i, (n, b) in enumerate(groups):
            q.channels[i] = int(n)
            q.bits[i] = int(b)
        return q


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "layers", "kv_heads", "q_heads", "head_dim", "rank_k", "rank_v", "window",
        "block", "max_tokens", "kv_dtype", "coef_dtype", "use_rope")] + [
        ("rope_theta", ctypes.c_double)] + [(n, ctypes.c_int32) for n in (
            "sync", "max_deferred", "jacobi_max_sweeps", "ring_extra", "protect",
            "coef_quant")] + [("quant_k", QuantFormat), ("quant_v", QuantFormat)] + [
        ("joint", ctypes.c_int32)]


class DecodeOperands(ctypes.Structure):
    """Mirror of ``iskv_decode_operands`` (allocation-free decode)."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "kv_heads", "q_heads", "head_dim", "rank_k", "rank_v", "kv_dtype",
        "coef_dtype")] + [(n, ctypes.c_int64) for n in ("T", "n_c", "coef_rows", "ring_rows")] + [
        (n, ctypes.c_void_p) for n in ("coef_k", "basis_k", "coef_v", "basis_v", "ring_k",
                                       "ring_v", "rope")]


_vp, _i, _i64p = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)
_SIGS = {
    "iskv_config_default": ([ctypes.POINTER(_Cfg)], _i),
    "iskv_create": ([ctypes.POINTER(_Cfg), _vp, ctypes.POINTER(_vp)], _i),
    "iskv_destroy": ([_vp], _i),
    "iskv_append": ([_vp, _i, _vp, _vp, _i, _vp, ctypes.POINTER(_i)], _i),
    "iskv_compress_block": ([_vp, _i, _i, _vp], _i),
    "iskv_sync": ([_vp, _i, _vp], _i),
    "iskv_decode_attention": ([_vp, _i, _vp, _vp, _vp], _i),
    "iskv_reconstruct": ([_vp, _i, _i, _vp, _vp], _i),
    "iskv_get_factors": ([_vp, _i, _i, _vp, _vp, _vp, _vp], _i),
    "iskv_get_counts": ([_vp, _i, _i64p, _i64p], _i),
    "iskv_kv_bytes": ([_vp, _i64p, _i64p], _i),
    "iskv_decode_kernel": ([_vp, _i, ctypes.POINTER(_i)], _i),
    "iskv_compress_block_async": ([_vp, _i, _i, _vp, _vp], _i),
    "iskv_status": ([_vp], _i),
    "iskv_strerror": ([_i], ctypes.c_char_p),
    "iskv_decode_attention_noalloc": ([ctypes.POINTER(DecodeOperands), _vp, _vp, _vp], _i),
    "iskv_quantize_rows": ([ctypes.POINTER(QuantFormat), _i, _vp, ctypes.c_int64, _vp, _vp, _vp], _i),
    "iskv_quant_words": ([ctypes.POINTER(QuantFormat)], _i),
}
for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(LIB, _name)
    _fn.argtypes = _args
    _fn.restype = _ret
EXPORTED = tuple(_SIGS)


def _check(code: int, where: str) -> None:
    if code != OK:
        raise IskvError(code, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_TORCH_DT = {F32: torch.float32, BF16: torch.bfloat16}


@dataclass
class Config:
    """Mirror of ``iskv_config``; defaults are the one-layer Qwen3-8B-shaped cache."""
    batch: int = 1
    layers: int = 1
    kv_heads: int = 8
    q_heads: int = 32
    head_dim: int = 128
    rank_k: int = 32
    rank_v: int = 64
    window: int = 1024
    block: int = 64
    max_tokens: int = 16384
    kv_dtype: int = BF16
    coef_dtype: int = F32
    use_rope: int = 1
    rope_theta: float = 1e6
    sync: int = 1
    max_deferred: int = 0
    jacobi_max_sweeps: int = 0
    ring_extra: int = 0
    protect: int = 0
    coef_quant: int = 0
    quant_k: tuple = ()        # ((channels, bits), ...) of the K factor's code groups
    quant_v: tuple = ()
    joint: int = 0             # 1: one factor per sequence over all KV heads (D = kv_heads*128)

    def _c(self) -> _Cfg:
        c = _Cfg()
        for f in _Cfg._fields_:
            if f[0] in ("quant_k", "quant_v"):
                groups = getattr(self, f[0])
                if groups:
                    setattr(c, f[0], QuantFormat.of(groups))
                continue
            setattr(c, f[0], getattr(self, f[0]))
        return c

    @property
    def kv_torch_dtype(self):
        return _TORCH_DT[self.kv_dtype]

    @property
    def coef_torch_dtype(self):
        return _TORCH_DT[self.coef_dtype]


class Cache:
    """One iS-KV cache (all layers of a batch).  Methods mirror the C ABI."""

    def __init__(self, cfg: Config, stream=None):
        self.cfg = cfg
        self._h = ctypes.c_void_p()
        self._cc = cfg._c()
        _check(LIB.iskv_create(ctypes.byref(self._cc), _stream(stream), ctypes.byref(self._h)),
               "iskv_create")

    def close(self) -> None:
        if getattr(self, "_h", None) and self._h.value:
            LIB.iskv_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def append(self, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> int:
        """k, v: [batch, kv_heads, t, d] pre-RoPE, device or host memory."""
        c = self.cfg
        if k.shape != v.shape or k.dim() != 4 or k.shape[:2] != (c.batch, c.kv_heads) \
                or k.shape[3] != c.head_dim:
            raise ValueError(f"k/v shape {tuple(k.shape)} does not match the cache")
        if k.dtype != c.kv_torch_dtype or v.dtype != c.kv_torch_dtype:
            raise TypeError("k/v dtype does not match kv_dtype")
        ready = ctypes.c_int(0)
        _check(LIB.iskv_append(self._h, layer, _ptr(k), _ptr(v), int(k.shape[2]), _stream(stream),
                               ctypes.byref(ready)), "iskv_append")
        return ready.value

    def compress_block(self, layer: int = ALL_LAYERS, defer: bool = False, stream=None) -> None:
        _check(LIB.iskv_compress_block(self._h, layer, FOLD_DEFER_SYNC if defer else 0,
                                       _stream(stream)), "iskv_compress_block")

    def compress_block_async(self, layer: int, stream, after=None, defer: bool = False) -> None:
        """The block update of `layer` on `stream` (a second stream), after the
        work enqueued so far on `after` (default: the current stream); later
        calls touching the layer are ordered after it by the library."""
        _check(LIB.iskv_compress_block_async(self._h, layer, FOLD_DEFER_SYNC if defer else 0,
                                             _stream(stream), _stream(after)),
               "iskv_compress_block_async")

    def sync(self, layer: int = ALL_LAYERS, stream=None) -> None:
        _check(LIB.iskv_sync(self._h, layer, _stream(stream)), "iskv_sync")

    def decode_attention(self, layer: int, q: torch.Tensor, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
        """q: [batch, q_heads, d] (rotated for position T-1); returns fp32 out."""
        c = self.cfg
        if tuple(q.shape) != (c.batch, c.q_heads, c.head_dim) or q.dtype != c.kv_torch_dtype:
            raise ValueError("q shape/dtype does not match the cache")
        if out is None:
            out = torch.empty(c.batch, c.q_heads, c.head_dim, dtype=torch.float32, device=q.device)
        _check(LIB.iskv_decode_attention(self._h, layer, _ptr(q), _ptr(out), _stream(stream)),
               "iskv_decode_attention")
        return out

    def reconstruct(self, layer: int, which: int, out: torch.Tensor | None = None,
                    stream=None, device="cuda") -> torch.Tensor:
        c = self.cfg
        n_c = self.counts(layer)[1]
        if out is None:
            out = torch.empty(c.batch, c.kv_heads, n_c, c.head_dim, dtype=torch.float32,
                              device=device)
        _check(LIB.iskv_reconstruct(self._h, layer, which, _ptr(out), _stream(stream)),
               "iskv_reconstruct")
        return out

    def factors(self, layer: int, which: int, stream=None, device="cuda"):
        """(basis [B,H,d,r] fp32, sigma [B,H,r] fp32, coef [B,H,n_c,r]); for a
        joint-head cache (basis [B,H*d,r], sigma [B,r], coef [B,n_c,r])."""
        c = self.cfg
        r = c.rank_k if which == WHICH_K else c.rank_v
        n_c = self.counts(layer)[1]
        cdt = torch.float32 if c.coef_quant else c.coef_torch_dtype   # coded: values code * scale
        if c.joint:
            basis = torch.empty(c.batch, c.kv_heads * c.head_dim, r, dtype=torch.float32, device=device)
            sigma = torch.empty(c.batch, r, dtype=torch.float32, device=device)
            coef = torch.empty(c.batch, n_c, r, dtype=cdt, device=device)
        else:
            basis = torch.empty(c.batch, c.kv_heads, c.head_dim, r, dtype=torch.float32, device=device)
            sigma = torch.empty(c.batch, c.kv_heads, r, dtype=torch.float32, device=device)
            coef = torch.empty(c.batch, c.kv_heads, n_c, r, dtype=cdt, device=device)
        _check(LIB.iskv_get_factors(self._h, layer, which, _ptr(basis), _ptr(sigma),
                                    _ptr(coef) if n_c else None, _stream(stream)),
               "iskv_get_factors")
        return basis, sigma, coef

    def counts(self, layer: int):
        T, n = ctypes.c_int64(), ctypes.c_int64()
        _check(LIB.iskv_get_counts(self._h, layer, ctypes.byref(T), ctypes.byref(n)),
               "iskv_get_counts")
        return T.value, n.value

    def kv_bytes(self):
        """(persistent bytes kept between decode steps, bytes of the uncompressed
        K/V cache at the same T), summed over every layer, sequence and KV head."""
        p, f = ctypes.c_int64(), ctypes.c_int64()
        _check(LIB.iskv_kv_bytes(self._h, ctypes.byref(p), ctypes.byref(f)), "iskv_kv_bytes")
        return p.value, f.value

    def decode_kernel(self, layer: int = 0) -> str:
        """The kernel the next decode_attention of `layer` runs: "cuda_core",
        "rotate" (tensor cores, keys rebuilt and rotated per tile) or
        "query_rope" (tensor cores, RoPE folded into the queries)."""
        k = _i()
        _check(LIB.iskv_decode_kernel(self._h, layer, ctypes.byref(k)), "iskv_decode_kernel")
        return {0: "cuda_core", 1: "rotate", 2: "query_rope"}[k.value]

    def status(self) -> int:
        return LIB.iskv_status(self._h)


def quantize_rows(groups, rows: torch.Tensor, stream=None):
    """Code fp32 rows [n, rank] (device) with the latent-channel format
    ``groups`` = ((channels, bits), ...): returns (codes [n, words] int32
    holding the uint32 words, scales [n, 4] fp32)."""
    fmt = QuantFormat.of(groups)
    words = LIB.iskv_quant_words(ctypes.byref(fmt))
    if words < 0:
        raise ValueError(f"invalid code format {groups}")
    if rows.dtype != torch.float32 or rows.dim() != 2:
        raise TypeError("rows must be a 2-d fp32 tensor")
    n, rank = rows.shape
    codes = torch.zeros(n, words, dtype=torch.int32, device=rows.device)
    scales = torch.zeros(n, 4, dtype=torch.float32, device=rows.device)
    _check(LIB.iskv_quantize_rows(ctypes.byref(fmt), rank, _ptr(rows), n, _ptr(codes), _ptr(scales),
                                  _stream(stream)), "iskv_quantize_rows")
    return codes, scales
