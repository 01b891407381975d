"""Python binding of libtq: TurboQuant-style K/V quantization and decode
attention from packed codes on an NVIDIA B200.

Argument marshalling only: every step runs in libtq's CUDA kernels.  PyTorch
supplies device memory (the tensors passed in, and the outputs this module
allocates for convenience) and the current CUDA stream.  There is no CPU
fallback: importing fails if libtq.so has not been built, and every call
raises TQError when the library reports an error.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
_LIB_PATH = _PKG / "libtq.so"

TQ_OK, TQ_ERR_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_WORKSPACE = range(5)
TQ_KEY, TQ_VALUE = 0, 1
TQ_NC_KEYS, TQ_NC_VALUES, TQ_NORM_F16 = 1, 2, 4
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2

_DTYPES = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}


class TQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libtq status {status}: {msg}")
        self.status = status


class tq_layout_t(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("bits", ctypes.c_int32), ("words", ctypes.c_int32),
                ("qjl_m", ctypes.c_int32), ("qjl_words", ctypes.c_int32),
                ("has_rnorm", ctypes.c_int32), ("bytes_per_vector", ctypes.c_int64),
                ("norm_bytes", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not _LIB_PATH.exists():
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m compressed_decode_attention_quantize_b200.build`")
    lib = ctypes.CDLL(str(_LIB_PATH))
    P, I, I64, U64, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                              ctypes.c_size_t, ctypes.c_float)
    sig = {
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_version": (ctypes.c_char_p, []),
        "tq_device_fault": (I, [ctypes.POINTER(ctypes.c_int)]),
        "tq_set_wait_limit": (I, [P, I]),
        "tq_init": (P, [I, I, I, I, U64]),
        "tq_init_ex": (P, [I, I, I, I, U64, I]),
        "tq_destroy": (None, [P]),
        "tq_layout": (I, [P, I, ctypes.POINTER(tq_layout_t)]),
        "tq_host_tables": (I, [I, I, I, I, U64, P, P, P, P, P, P]),
        "tq_export_tables": (I, [P, P, P, P, P, P, P]),
        "tq_quantize": (I, [P, I, P, I, I64, I64, P, P, P, P, P]),
        "tq_quantize_append": (I, [P, I, P, I, I, I, I64, I64, P, P, P, P, P, P]),
        "tq_dequantize": (I, [P, I, P, P, P, P, I64, P, P]),
        "tq_logits": (I, [P, P, I, I64, P, P, P, P, I64, P, P]),
        "tq_attn_workspace_bytes": (SZ, [P, I, I, I64]),
        "tq_attn_decode": (I, [P, P, I, I, I, I, P, P, P, P, P, P, I64, P, F, P, P, SZ, P]),
        "tq_attn_decode_static": (I, [P, P, I, I, I, I, P, P, P, P, P, P, I64, P, F, P, P]),
        "tq_attn_static_scratch_bytes": (SZ, []),
        "tq_decode_step": (I, [P, P, I, P, P, I, I, I, I, P, P, P, P, P, P, I64, P, F, P, P, SZ, P]),
        "tq_quantize_append_paged": (I, [P, I, P, I, I, I, I64, P, I, I, I64, P, P, P, P, P, P]),
        "tq_attn_decode_paged": (I, [P, P, I, I, I, I, P, P, P, P, P, P, P, I, I, I64, P, F, P, P, SZ, P]),
        "tq_decode_step_paged": (I, [P, P, I, P, P, I, I, I, I, P, P, P, P, P, P, P, I, I, I64, P, F, P, P,
                                     SZ, P]),
        "tq_topk_workspace_bytes": (SZ, [P, I64, I64, I]),
        "tq_topk": (I, [P, P, I, I64, P, P, P, P, I64, I, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("tq_last_error", "tq_version", "tq_device_fault", "tq_set_wait_limit", "tq_init", "tq_init_ex", "tq_destroy", "tq_layout", "tq_host_tables",
            "tq_export_tables", "tq_quantize", "tq_quantize_append", "tq_dequantize", "tq_logits",
            "tq_attn_workspace_bytes", "tq_attn_decode", "tq_attn_decode_static",
            "tq_attn_static_scratch_bytes", "tq_decode_step", "tq_quantize_append_paged",
            "tq_attn_decode_paged", "tq_decode_step_paged", "tq_topk_workspace_bytes", "tq_topk")


def library_path() -> str:
    return str(_LIB_PATH)


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TQError(status, _lib.tq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------
# Raw C-ABI wrappers (same names as the C entry points; pointers as ints or
# ctypes values).  The Context class below builds on them.
# ---------------------------------------------------------------------------
def tq_init(d, bits_k, bits_v, qjl_m, seed):
    p = _lib.tq_init(d, bits_k, bits_v, qjl_m, seed)
    if not p:
        raise TQError(-1, _lib.tq_last_error().decode())
    return p


def tq_init_ex(d, bits_k, bits_v, qjl_m, seed, flags):
    p = _lib.tq_init_ex(d, bits_k, bits_v, qjl_m, seed, flags)
    if not p:
        raise TQError(-1, _lib.tq_last_error().decode())
    return p


def tq_destroy(ctx):
    _lib.tq_destroy(ctx)


def tq_device_fault() -> int:
    """Read and clear the device fault code (0 = none); synchronises."""
    v = ctypes.c_int(0)
    _check(_lib.tq_device_fault(ctypes.byref(v)))
    return v.value


def tq_set_wait_limit(ctx, polls: int) -> None:
    """Test diagnostic: the context's tensor-core kernels give up their main
    bounded waits after `polls` polls (0 = the full limit)."""
    _check(_lib.tq_set_wait_limit(ctx, polls))


def tq_version() -> str:
    return _lib.tq_version().decode()


def tq_layout(ctx, which) -> dict:
    out = tq_layout_t()
    _check(_lib.tq_layout(ctx, which, ctypes.byref(out)))
    return {f: getattr(out, f) for f, _ in tq_layout_t._fields_}


def tq_host_tables(d, bits_k, bits_v, qjl_m, seed):
    """Tables computed by the library's host code (no GPU needed), fp64 numpy."""
    import numpy as np
    bk_lm = bits_k - 1 if qjl_m > 0 else bits_k
    pi = np.zeros((d, d))
    S = np.zeros((max(qjl_m, 1), d))
    ck = np.zeros(1 << bk_lm)
    bk = np.zeros((1 << bk_lm) - 1)
    cv = np.zeros(1 << bits_v)
    bv = np.zeros((1 << bits_v) - 1)
    args = [a.ctypes.data_as(ctypes.c_void_p) for a in (pi, S, ck, bk, cv, bv)]
    _check(_lib.tq_host_tables(d, bits_k, bits_v, qjl_m, seed, *args))
    return {"Pi": pi, "S": S[:qjl_m], "ck": ck, "bk": bk, "cv": cv, "bv": bv}


# Named cache formats: name -> (bits_k, bits_v, key QJL stage with m = d,
# norm correction of keys and values).  k3v4 / k4v4 spend one key bit on QJL;
# the _nc formats of the vLLM study are MSE-only with norm correction, and
# k8v4 has MSE-only 8-bit keys.
VARIANTS = {
    "k3v4": (3, 4, True, False),
    "k4v4": (4, 4, True, False),
    "k3v4_nc": (3, 4, False, True),
    "4bit_nc": (4, 4, False, True),
    "3bit_nc": (3, 3, False, True),
    "k8v4": (8, 4, False, False),
}


class Context:
    """A libtq context: tables for one (d, bits_k, bits_v, qjl_m, seed) on the
    current CUDA device."""

    def __init__(self, d: int, bits_k: int, bits_v: int, qjl_m: int, seed: int = 0,
                 nc_k: bool = False, nc_v: bool = False, norm_f16: bool = False):
        self.d, self.bits_k, self.bits_v, self.qjl_m, self.seed = d, bits_k, bits_v, qjl_m, seed
        self.nc_k, self.nc_v, self.norm_f16 = bool(nc_k), bool(nc_v), bool(norm_f16)
        flags = ((TQ_NC_KEYS if nc_k else 0) | (TQ_NC_VALUES if nc_v else 0) |
                 (TQ_NORM_F16 if norm_f16 else 0))
        self.ptr = tq_init_ex(d, bits_k, bits_v, qjl_m, seed, flags)
        self.key_layout = tq_layout(self.ptr, TQ_KEY)
        self.value_layout = tq_layout(self.ptr, TQ_VALUE)

    @classmethod
    def variant(cls, name: str, d: int, seed: int = 0, norm_f16: bool = False) -> "Context":
        """A context for one of the named cache formats in VARIANTS; norm_f16
        stores the norms as binary16 (formats without QJL)."""
        if name not in VARIANTS:
            raise ValueError(f"unknown variant {name!r}; known: {', '.join(VARIANTS)}")
        bits_k, bits_v, qjl, nc = VARIANTS[name]
        return cls(d, bits_k, bits_v, d if qjl else 0, seed, nc_k=nc, nc_v=nc, norm_f16=norm_f16)

    def set_wait_limit(self, polls: int) -> None:
        """Test diagnostic (tq_set_wait_limit): main bounded waits of this
        context's tensor-core kernels give up after `polls` polls; 0 restores
        the full limit."""
        tq_set_wait_limit(self.ptr, polls)

    def close(self):
        if getattr(self, "ptr", None):
            tq_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layout(self, which: int) -> dict:
        return self.key_layout if which == TQ_KEY else self.value_layout

    def _norm(self, which: int, packed: dict):
        """The packed dict's norm array, refused unless it holds this
        context's norm type (fp32, or binary16 under TQ_NORM_F16): the C ABI
        takes norms as untyped pointers and cannot tell them apart."""
        t = packed["norm"]
        want = torch.float16 if self.layout(which)["norm_bytes"] == 2 else torch.float32
        if t.dtype != want:
            raise TQError(TQ_ERR_ARG, f"norm array of dtype {t.dtype}; this context stores {want} norms")
        return t

    def tables(self):
        import numpy as np
        d, kl = self.d, self.key_layout
        pi = np.zeros((d, d))
        S = np.zeros((max(self.qjl_m, 1), d))
        ck = np.zeros(1 << kl["bits"])
        bk = np.zeros((1 << kl["bits"]) - 1)
        cv = np.zeros(1 << self.bits_v)
        bv = np.zeros((1 << self.bits_v) - 1)
        args = [a.ctypes.data_as(ctypes.c_void_p) for a in (pi, S, ck, bk, cv, bv)]
        _check(_lib.tq_export_tables(self.ptr, *args))
        return {"Pi": pi, "S": S[:self.qjl_m], "ck": ck, "bk": bk, "cv": cv, "bv": bv}

    # -- storage -------------------------------------------------------------
    def empty_packed(self, which: int, lead_shape, device="cuda") -> dict:
        """Caller-owned packed arrays for vectors of shape lead_shape."""
        L = self.layout(which)
        lead = tuple(lead_shape)
        out = {
            "codes": torch.empty(lead + (L["words"],), dtype=torch.int32, device=device),
            "norm": torch.empty(lead, dtype=torch.float16 if L["norm_bytes"] == 2 else torch.float32,
                                device=device),
            "qjl": None, "rnorm": None,
        }
        if L["has_rnorm"]:
            out["qjl"] = torch.empty(lead + (L["qjl_words"],), dtype=torch.int32, device=device)
            out["rnorm"] = torch.empty(lead, dtype=torch.float32, device=device)
        return out

    # -- operations ----------------------------------------------------------
    def quantize_into(self, x: torch.Tensor, which: int, packed: dict, stream=None) -> dict:
        x2 = x.reshape(-1, x.shape[-1])
        if x2.stride(-1) != 1:
            raise TQError(TQ_ERR_ARG, "x must have a unit inner stride")
        n = x2.shape[0]
        _check(_lib.tq_quantize(self.ptr, which, _ptr(x2), _DTYPES[x.dtype], n, x2.stride(0),
                                _ptr(packed["codes"]), _ptr(packed["qjl"]), _ptr(self._norm(which, packed)),
                                _ptr(packed["rnorm"]), _stream(stream)))
        return packed

    def quantize(self, x: torch.Tensor, which: int, stream=None) -> dict:
        packed = self.empty_packed(which, x.shape[:-1], device=x.device)
        return self.quantize_into(x, which, packed, stream)

    def quantize_append(self, x: torch.Tensor, which: int, cache: dict, pos: torch.Tensor,
                        stream=None) -> dict:
        """x [B, H, d] (newest token per sequence and head) -> cache[b, g, pos[b]]."""
        B, H, d = x.shape
        if x.stride(2) != 1 or x.stride(0) != H * x.stride(1):
            raise TQError(TQ_ERR_ARG, "x must be [B, H, d] with rows at a uniform stride")
        max_T = cache["norm"].shape[2]
        _check(_lib.tq_quantize_append(self.ptr, which, _ptr(x), _DTYPES[x.dtype], B, H,
                                       x.stride(1), max_T, _ptr(pos), _ptr(cache["codes"]),
                                       _ptr(cache["qjl"]), _ptr(self._norm(which, cache)), _ptr(cache["rnorm"]),
                                       _stream(stream)))
        return cache

    def dequantize(self, which: int, packed: dict, out: torch.Tensor | None = None, stream=None):
        n = packed["norm"].numel()
        if out is None:
            out = torch.empty(packed["norm"].shape + (self.d,), dtype=torch.float32,
                              device=packed["norm"].device)
        _check(_lib.tq_dequantize(self.ptr, which, _ptr(packed["codes"]), _ptr(packed["qjl"]),
                                  _ptr(self._norm(which, packed)), _ptr(packed["rnorm"]), n, _ptr(out),
                                  _stream(stream)))
        return out

    def logits(self, q: torch.Tensor, keys: dict, out: torch.Tensor | None = None, stream=None):
        q2 = q.reshape(-1, self.d).contiguous()
        nk = keys["norm"].numel()
        if out is None:
            out = torch.empty(q2.shape[0], nk, dtype=torch.float32, device=q.device)
        _check(_lib.tq_logits(self.ptr, _ptr(q2), _DTYPES[q.dtype], q2.shape[0],
                              _ptr(keys["codes"]), _ptr(keys["qjl"]), _ptr(self._norm(TQ_KEY, keys)),
                              _ptr(keys["rnorm"]), nk, _ptr(out), _stream(stream)))
        return out

    def attn_workspace_bytes(self, B: int, Hq: int, max_T: int) -> int:
        return int(_lib.tq_attn_workspace_bytes(self.ptr, B, Hq, max_T))

    def attn_decode(self, q: torch.Tensor, kcache: dict, vcache: dict, seq_lens: torch.Tensor,
                    scale: float | None = None, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """q [B, Hq, d]; caches as dicts of [B, Hkv, max_T, ...] arrays."""
        q = q.contiguous()
        B, Hq, d = q.shape
        Hkv, max_T = kcache["norm"].shape[1], kcache["norm"].shape[2]
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        need = self.attn_workspace_bytes(B, Hq, max_T)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _check(_lib.tq_attn_decode(self.ptr, _ptr(q), _DTYPES[q.dtype], B, Hq, Hkv,
                                   _ptr(kcache["codes"]), _ptr(kcache["qjl"]), _ptr(self._norm(TQ_KEY, kcache)),
                                   _ptr(kcache["rnorm"]), _ptr(vcache["codes"]), _ptr(self._norm(TQ_VALUE, vcache)),
                                   max_T, _ptr(seq_lens), float(scale), _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))
        return out

    def decode_step(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, kcache: dict,
                    vcache: dict, pos: torch.Tensor, scale: float | None = None,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
        """Append k_new / v_new [B, Hkv, d] at slot pos[b] of the caches, then
        attend q [B, Hq, d] over tokens [0, pos[b]] (tq_decode_step)."""
        q, k_new, v_new = q.contiguous(), k_new.contiguous(), v_new.contiguous()
        B, Hq, d = q.shape
        Hkv, max_T = kcache["norm"].shape[1], kcache["norm"].shape[2]
        if k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d) or k_new.dtype != v_new.dtype:
            raise TQError(TQ_ERR_ARG, "decode_step: k_new / v_new must both be [B, Hkv, d] of one dtype")
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        need = self.attn_workspace_bytes(B, Hq, max_T)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _check(_lib.tq_decode_step(self.ptr, _ptr(q), _DTYPES[q.dtype], _ptr(k_new), _ptr(v_new),
                                   _DTYPES[k_new.dtype], B, Hq, Hkv, _ptr(kcache["codes"]),
                                   _ptr(kcache["qjl"]), _ptr(self._norm(TQ_KEY, kcache)), _ptr(kcache["rnorm"]),
                                   _ptr(vcache["codes"]), _ptr(self._norm(TQ_VALUE, vcache)), max_T, _ptr(pos),
                                   float(scale), _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))
        return out

    # ---- paged caches: arrays [num_blocks, Hkv, block_size, ...] (empty_packed
    # with that shape), block_table int32 [B, max_blocks] of block ids --------
    def quantize_append_paged(self, x: torch.Tensor, which: int, cache: dict, block_table: torch.Tensor,
                              pos: torch.Tensor, stream=None) -> dict:
        """x [B, H, d] (newest token per sequence and head) -> the slot of
        position pos[b] in block block_table[b, pos[b] // block_size]."""
        B, H, d = x.shape
        if x.stride(2) != 1 or x.stride(0) != H * x.stride(1):
            raise TQError(TQ_ERR_ARG, "x must be [B, H, d] with rows at a uniform stride")
        nb, _, bs = cache["norm"].shape
        _check(_lib.tq_quantize_append_paged(self.ptr, which, _ptr(x), _DTYPES[x.dtype], B, H, x.stride(1),
                                             _ptr(block_table), block_table.shape[1], bs, nb, _ptr(pos),
                                             _ptr(cache["codes"]), _ptr(cache.get("qjl")),
                                             _ptr(self._norm(which, cache)), _ptr(cache.get("rnorm")), _stream(stream)))
        return cache

    def attn_decode_paged(self, q: torch.Tensor, kcache: dict, vcache: dict, block_table: torch.Tensor,
                          seq_lens: torch.Tensor, scale: float | None = None,
                          out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
        q = q.contiguous()
        B, Hq, d = q.shape
        nb, Hkv, bs = kcache["norm"].shape
        mb = block_table.shape[1]
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(self.attn_workspace_bytes(B, Hq, mb * bs), dtype=torch.uint8,
                                    device=q.device)
        _check(_lib.tq_attn_decode_paged(self.ptr, _ptr(q), _DTYPES[q.dtype], B, Hq, Hkv,
                                         _ptr(kcache["codes"]), _ptr(kcache["qjl"]), _ptr(self._norm(TQ_KEY, kcache)),
                                         _ptr(kcache["rnorm"]), _ptr(vcache["codes"]), _ptr(self._norm(TQ_VALUE, vcache)),
                                         _ptr(block_table), mb, bs, nb, _ptr(seq_lens), float(scale),
                                         _ptr(out), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
        return out

    def decode_step_paged(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                          kcache: dict, vcache: dict, block_table: torch.Tensor, pos: torch.Tensor,
                          scale: float | None = None, out: torch.Tensor | None = None,
                          workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        q, k_new, v_new = q.contiguous(), k_new.contiguous(), v_new.contiguous()
        B, Hq, d = q.shape
        nb, Hkv, bs = kcache["norm"].shape
        mb = block_table.shape[1]
        if k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d) or k_new.dtype != v_new.dtype:
            raise TQError(TQ_ERR_ARG, "decode_step_paged: k_new / v_new must both be [B, Hkv, d] of one dtype")
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(self.attn_workspace_bytes(B, Hq, mb * bs), dtype=torch.uint8,
                                    device=q.device)
        _check(_lib.tq_decode_step_paged(self.ptr, _ptr(q), _DTYPES[q.dtype], _ptr(k_new), _ptr(v_new),
                                         _DTYPES[k_new.dtype], B, Hq, Hkv, _ptr(kcache["codes"]),
                                         _ptr(kcache["qjl"]), _ptr(self._norm(TQ_KEY, kcache)), _ptr(kcache["rnorm"]),
                                         _ptr(vcache["codes"]), _ptr(self._norm(TQ_VALUE, vcache)), _ptr(block_table), mb,
                                         bs, nb, _ptr(pos), float(scale), _ptr(out), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
        return out

    def attn_decode_static(self, q: torch.Tensor, kcache: dict, vcache: dict,
                           seq_lens: torch.Tensor, scale: float | None = None,
                           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """attn_decode using the library's static device scratch instead of a
        workspace (for callers that cannot allocate); calls must not overlap."""
        q = q.contiguous()
        B, Hq, d = q.shape
        Hkv, max_T = kcache["norm"].shape[1], kcache["norm"].shape[2]
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        _check(_lib.tq_attn_decode_static(self.ptr, _ptr(q), _DTYPES[q.dtype], B, Hq, Hkv,
                                          _ptr(kcache["codes"]), _ptr(kcache["qjl"]),
                                          _ptr(self._norm(TQ_KEY, kcache)), _ptr(kcache["rnorm"]),
                                          _ptr(vcache["codes"]), _ptr(self._norm(TQ_VALUE, vcache)), max_T,
                                          _ptr(seq_lens), float(scale), _ptr(out), _stream(stream)))
        return out

    def topk_workspace_bytes(self, nq: int, n: int, k: int) -> int:
        return int(_lib.tq_topk_workspace_bytes(self.ptr, nq, n, k))

    def topk(self, q: torch.Tensor, db: dict, k: int, workspace: torch.Tensor | None = None,
             stream=None):
        q2 = q.reshape(-1, self.d).contiguous()
        nq, n = q2.shape[0], db["norm"].numel()
        idx = torch.empty(nq, k, dtype=torch.int32, device=q.device)
        score = torch.empty(nq, k, dtype=torch.float32, device=q.device)
        need = self.topk_workspace_bytes(nq, n, k)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _check(_lib.tq_topk(self.ptr, _ptr(q2), _DTYPES[q.dtype], nq, _ptr(db["codes"]),
                            _ptr(db["qjl"]), _ptr(self._norm(TQ_KEY, db)), _ptr(db["rnorm"]), n, k, _ptr(idx),
                            _ptr(score), _ptr(workspace), workspace.numel(), _stream(stream)))
        return idx, score
