"""Python binding of the DeltaLog C ABI (``include/deltalog.h``).

Argument marshalling only: every function here has the name of the C entry
point it calls and passes plain device pointers, sizes and a CUDA stream
through ctypes.  All arithmetic runs in the CUDA kernels of
``libdeltalog.so``.  Torch tensors are accepted as the carriers of device
memory (their ``data_ptr()``); the binding checks their dtype, device, size
and contiguity so that the C library never sees a buffer smaller than the
layout it is told about.

Importing this module loads the library and fails loudly when it has not
been built (``python -m linear_attention_recurrent_deltalog_b200.build``):
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdeltalog.so")

# enums (mirror deltalog.h)
DL_GDN, DL_KDA, DL_RWKV6, DL_GDN2 = 0, 1, 2, 3
DL_F32, DL_BF16 = 0, 1
DL_OK = 0
DL_ERR_ARG, DL_ERR_ALIGN, DL_ERR_LOG_FULL = -1, -2, -3
DL_ERR_CUDA, DL_ERR_UNSUPPORTED, DL_ERR_DEVICE = -4, -5, -6
DL_MERGE_FULL, DL_MERGE_ALL = 0, 1
DL_FLAG_FUSED_MERGE = 1
DL_FLAG_KLA = 4
DL_FLAG_BASE_Q8 = 8

VARIANT_IDS = {"gdn": DL_GDN, "kda": DL_KDA, "rwkv6": DL_RWKV6, "gdn2": DL_GDN2}
DTYPE_IDS = {"f32": DL_F32, "bf16": DL_BF16}
_TORCH_IN = {DL_F32: torch.float32, DL_BF16: torch.bfloat16}


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -m linear_attention_recurrent_deltalog_b200.build` (there is no CPU fallback)")
    return ctypes.CDLL(_LIB_PATH)


_lib = _load()


class dl_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("variant", "B", "H", "d_k", "d_v", "L", "in_dtype", "flags", "step_split")] + \
        [("kla_eps", ctypes.c_float)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.POINTER(ctypes.c_size_t)
_CFG = ctypes.POINTER(dl_config)

_SIGS = {
    "dl_state_bytes": (_I, [_CFG, _SZ, _SZ, _SZ]),
    "dl_state_create": (_I, [_CFG, _P, _P, _P, ctypes.POINTER(_P)]),
    "dl_state_reset": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int32), _P]),
    "dl_state_load_seqs": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int32), _P, _P]),
    "dl_decode_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_merge": (_I, [_P, _I, _P]),
    "dl_materialize": (_I, [_P, _P, _P]),
    "dl_eager_step": (_I, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_state_fill": (_I, [_P, ctypes.POINTER(ctypes.c_int32)]),
    "dl_state_destroy": (_I, [_P]),
    "dl_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                             _I, _P]),
    "dl_selftest_wait_timeout": (_I, [ctypes.POINTER(ctypes.c_int32), _P]),
    "dl_launch_count": (ctypes.c_uint64, []),
    "dl_status_string": (ctypes.c_char_p, [_I]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)
LIB_PATH = _LIB_PATH


class DeltaLogError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {dl_status_string(status)} ({status})")


def _check(status: int, call: str) -> int:
    if status < 0:
        raise DeltaLogError(status, call)
    return status


def dl_status_string(status: int) -> str:
    return _lib.dl_status_string(int(status)).decode()


def dl_launch_count() -> int:
    return int(_lib.dl_launch_count())


def dl_selftest_wait_timeout(stream=None) -> int:
    """Runs the bounded-wait failure path once; returns the recorded code."""
    code = ctypes.c_int32()
    _check(_lib.dl_selftest_wait_timeout(ctypes.byref(code), _stream(stream)),
           "dl_selftest_wait_timeout")
    return code.value


# ----------------------------------------------------------------- config

@dataclasses.dataclass(frozen=True)
class Config:
    """Python mirror of ``dl_config``."""

    variant: str
    B: int
    H: int
    d_k: int
    d_v: int
    L: int
    in_dtype: str = "bf16"
    fused_merge: bool = False
    step_split: int = 0
    kla_eps: Optional[float] = None  # set: beta carries the KLA gate eta
    base: str = "f32"                # "f32", or "q8": int8 codes + row scales

    def c(self) -> dl_config:
        if self.base not in ("f32", "q8"):
            raise ValueError(f"base must be 'f32' or 'q8', not {self.base!r}")
        flags = (DL_FLAG_FUSED_MERGE if self.fused_merge else 0) | \
            (DL_FLAG_KLA if self.kla_eps is not None else 0) | \
            (DL_FLAG_BASE_Q8 if self.base == "q8" else 0)
        return dl_config(VARIANT_IDS[self.variant], self.B, self.H, self.d_k, self.d_v, self.L,
                         DTYPE_IDS[self.in_dtype], flags, self.step_split,
                         0.0 if self.kla_eps is None else float(self.kla_eps))

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def torch_in_dtype(self) -> torch.dtype:
        return _TORCH_IN[DTYPE_IDS[self.in_dtype]]


# ----------------------------------------------------------------- marshalling

def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, name: str, numel: int, dtype: torch.dtype) -> None:
    """Buffer checks that keep every kernel access inside the tensor."""
    if t is None or isinstance(t, int):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, need {numel}")


def _check_step_tensors(cfg: Config, q, k, v, decay, beta, bonus, o) -> None:
    BH, dk, dv = cfg.heads, cfg.d_k, cfg.d_v
    tin = cfg.torch_in_dtype
    _need(q, "q", BH * dk, tin)
    _need(k, "k", BH * dk, tin)
    _need(v, "v", BH * dv, tin)
    _need(decay, "decay", BH * (1 if cfg.variant == "gdn" else dk), torch.float32)
    if cfg.variant == "rwkv6":
        _need(bonus, "bonus", cfg.H * dk, torch.float32)
    elif cfg.variant == "gdn2":           # beta: erase gate; bonus: write gate
        _need(beta, "beta", BH * dk, torch.float32)
        _need(bonus, "bonus", BH * dv, torch.float32)
    else:
        _need(beta, "beta", BH, torch.float32)
    _need(o, "o", BH * dv, torch.float32)


# ----------------------------------------------------------------- C entry points

def dl_state_bytes(cfg: Config):
    """-> (base_bytes, log_bytes, meta_bytes)"""
    b, l, m = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    c = cfg.c()
    _check(_lib.dl_state_bytes(ctypes.byref(c), ctypes.byref(b), ctypes.byref(l), ctypes.byref(m)),
           "dl_state_bytes")
    return b.value, l.value, m.value


def dl_state_create(cfg: Config, base, log, meta) -> int:
    sizes = dl_state_bytes(cfg)
    for t, n, name in zip((base, log, meta), sizes, ("base", "log", "meta")):
        if isinstance(t, torch.Tensor) and t.numel() * t.element_size() < n:
            raise ValueError(f"{name}: {t.numel() * t.element_size()} bytes, need {n}")
    h = _P()
    c = cfg.c()
    _check(_lib.dl_state_create(ctypes.byref(c), _ptr(base), _ptr(log), _ptr(meta),
                                ctypes.byref(h)), "dl_state_create")
    return h.value


def dl_state_reset(handle: int, cfg: Config, S0=None, fill0: Optional[Sequence[int]] = None,
                   stream=None) -> None:
    _need(S0, "S0", cfg.heads * cfg.d_v * cfg.d_k, torch.float32)
    arr = None
    if fill0 is not None:
        if len(fill0) != cfg.B:
            raise ValueError("fill0 must have B entries")
        arr = (ctypes.c_int32 * cfg.B)(*[int(x) for x in fill0])
    _check(_lib.dl_state_reset(handle, _ptr(S0), arr, _stream(stream)), "dl_state_reset")


def dl_state_load_seqs(handle: int, cfg: Config, seqs: Sequence[int], S=None, stream=None) -> None:
    n = len(seqs)
    _need(S, "S", n * cfg.H * cfg.d_v * cfg.d_k, torch.float32)
    arr = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in seqs])
    _check(_lib.dl_state_load_seqs(handle, n, arr, _ptr(S), _stream(stream)), "dl_state_load_seqs")


def dl_decode_step(handle: int, cfg: Config, q, k, v, decay, beta, bonus, o, stream=None) -> None:
    _check_step_tensors(cfg, q, k, v, decay, beta, bonus, o)
    _check(_lib.dl_decode_step(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(beta),
                               _ptr(bonus), _ptr(o), _stream(stream)), "dl_decode_step")


def dl_merge(handle: int, mode: int = DL_MERGE_FULL, stream=None) -> None:
    _check(_lib.dl_merge(handle, int(mode), _stream(stream)), "dl_merge")


def dl_materialize(handle: int, cfg: Config, S_out, stream=None) -> None:
    _need(S_out, "S_out", cfg.heads * cfg.d_v * cfg.d_k, torch.float32)
    _check(_lib.dl_materialize(handle, _ptr(S_out), _stream(stream)), "dl_materialize")


def dl_eager_step(cfg: Config, S, q, k, v, decay, beta, bonus, o, stream=None) -> None:
    _need(S, "S", cfg.heads * cfg.d_v * cfg.d_k, torch.float32)
    _check_step_tensors(cfg, q, k, v, decay, beta, bonus, o)
    c = cfg.c()
    _check(_lib.dl_eager_step(ctypes.byref(c), _ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(decay),
                              _ptr(beta), _ptr(bonus), _ptr(o), _stream(stream)), "dl_eager_step")


def dl_state_fill(handle: int, cfg: Config):
    arr = (ctypes.c_int32 * cfg.B)()
    _check(_lib.dl_state_fill(handle, arr), "dl_state_fill")
    return list(arr)


def dl_state_destroy(handle: Optional[int]) -> None:
    _check(_lib.dl_state_destroy(handle), "dl_state_destroy")


def dl_device_error(handle: Optional[int], clear: bool = False, stream=None):
    code, head = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.dl_device_error(handle, ctypes.byref(code), ctypes.byref(head), int(clear),
                                _stream(stream)), "dl_device_error")
    return code.value, head.value


# ----------------------------------------------------------------- convenience

class DeltaLogState:
    """A state whose three buffers are torch device tensors (allocation is
    torch's; the library only borrows them)."""

    def __init__(self, cfg: Config, device="cuda"):
        self.cfg = cfg
        nb, nl, nm = dl_state_bytes(cfg)
        self.base = torch.empty(nb // 4, dtype=torch.float32, device=device)
        self.log = torch.empty(nl, dtype=torch.uint8, device=device)
        self.meta = torch.empty(nm, dtype=torch.uint8, device=device)
        self.handle = dl_state_create(cfg, self.base, self.log, self.meta)

    def reset(self, S0=None, fill0=None, stream=None) -> None:
        dl_state_reset(self.handle, self.cfg, S0, fill0, stream)

    def load_seqs(self, seqs, S=None, stream=None) -> None:
        dl_state_load_seqs(self.handle, self.cfg, seqs, S, stream)

    def step(self, q, k, v, decay, beta=None, bonus=None, o=None, stream=None):
        if o is None:
            o = torch.empty(self.cfg.heads * self.cfg.d_v, dtype=torch.float32, device=self.base.device)
        dl_decode_step(self.handle, self.cfg, q, k, v, decay, beta, bonus, o, stream)
        return o

    def merge(self, mode: int = DL_MERGE_FULL, stream=None) -> None:
        dl_merge(self.handle, mode, stream)

    def materialize(self, out=None, stream=None):
        if out is None:
            out = torch.empty(self.cfg.heads * self.cfg.d_v * self.cfg.d_k, dtype=torch.float32,
                              device=self.base.device)
        dl_materialize(self.handle, self.cfg, out, stream)
        return out

    def fill(self):
        return dl_state_fill(self.handle, self.cfg)

    # An int8 base in the layout deltalog.h documents: codes [B*H, d_v, d_k]
    # with each row's 16-byte chunks stored XOR-swizzled (chunk ^ (row mod 8)
    # for d_k = 128, chunk ^ ((row / 2) mod 4) for d_k = 64), then the fp32
    # row scales [B*H, d_v] at the next 256-byte boundary.
    def _scale_offset(self) -> int:
        n = self.cfg.heads * self.cfg.d_v * self.cfg.d_k
        return (n + 255) // 256 * 256

    def _q8_perm(self) -> torch.Tensor:
        """Physical position of each logical (row, c) code within a head."""
        if getattr(self, "_perm", None) is None:
            dv, dk = self.cfg.d_v, self.cfg.d_k
            r = torch.arange(dv).view(dv, 1)
            c = torch.arange(dk).view(1, dk)
            sw = (r & 7) if dk == 128 else ((r >> 1) & 3)
            self._perm = (r * dk + (((c >> 4) ^ sw) << 4) + (c & 15)).reshape(-1).to(self.base.device)
        return self._perm

    def base_codes_raw(self) -> torch.Tensor:
        """The stored int8 codes [B*H, d_v*d_k] in their swizzled order (a view)."""
        if self.cfg.base != "q8":
            raise ValueError("base_codes_raw: the base is fp32")
        c = self.cfg
        return self.base.view(torch.uint8)[:c.heads * c.d_v * c.d_k].view(torch.int8).view(
            c.heads, c.d_v * c.d_k)

    def base_codes(self, heads=None) -> torch.Tensor:
        """The codes of `heads` (all when None) in logical order [n, d_v, d_k] (a copy)."""
        raw = self.base_codes_raw()
        if heads is not None:
            raw = raw.index_select(0, torch.as_tensor(heads, device=raw.device))
        return raw[:, self._q8_perm()].view(-1, self.cfg.d_v, self.cfg.d_k)

    def set_base_codes(self, heads, codes: torch.Tensor) -> None:
        """Writes logical-order codes [n, d_v, d_k] of `heads` into the base."""
        raw = self.base_codes_raw()
        heads = torch.as_tensor(heads, device=raw.device)
        tmp = torch.empty((heads.numel(), raw.shape[1]), dtype=torch.int8, device=raw.device)
        tmp[:, self._q8_perm()] = codes.reshape(heads.numel(), -1).to(device=raw.device,
                                                                      dtype=torch.int8)
        raw.index_copy_(0, heads, tmp)

    def base_scales(self) -> torch.Tensor:
        """The fp32 row scales [B*H, d_v] (a view)."""
        if self.cfg.base != "q8":
            raise ValueError("base_scales: the base is fp32")
        c = self.cfg
        off = self._scale_offset()
        raw = self.base.view(torch.uint8)
        return raw[off:off + c.heads * c.d_v * 4].view(torch.float32).view(c.heads, c.d_v)

    def device_error(self, clear: bool = False, stream=None):
        return dl_device_error(self.handle, clear, stream)

    def close(self) -> None:
        if self.handle is not None:
            dl_state_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
