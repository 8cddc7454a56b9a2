"""Thin Python binding of the C ABI in include/rotate_attn.h.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``librotate_attn.so``.  PyTorch supplies device memory and the current CUDA
stream.  There is no fallback: if the library is missing or a call fails, a
``RotateAttnError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
# RA_LIBRARY=bounds loads the bounds-checked test build instead (the same
# ABI; every computed device index is checked, violations are reported as
# RA_ERR_DEVICE_BOUNDS by ra_check_device_error).
LIB_PATH = os.path.join(PKG, "librotate_attn_bounds.so" if os.environ.get("RA_LIBRARY") == "bounds"
                        else "librotate_attn.so")

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_WORKSPACE, RA_ERR_CUDA, \
    RA_ERR_DEVICE_TIMEOUT, RA_ERR_DEVICE_BOUNDS = range(7)
ROT = {"none": 0, "interleaved": 1, "half": 2, "full": 3, "blocks_interleaved": 4, "blocks_half": 5}
P_MODE = {"range": 0, "symmetric": 1}       # ra_p_mode


class RotateAttnError(RuntimeError):
    def __init__(self, call: str, status: int, detail: str):
        super().__init__(f"{call}: {status_string(status)} ({detail})")
        self.status = status


class Problem(ctypes.Structure):
    """Mirror of ra_problem."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("F", ctypes.c_int), ("Hh", ctypes.c_int), ("W", ctypes.c_int),
                ("n_text", ctypes.c_int), ("split", ctypes.c_int * 3),
                ("theta", ctypes.c_double), ("rot", ctypes.c_int), ("p_mode", ctypes.c_int),
                ("v_rot", ctypes.c_int), ("blocks", ctypes.c_void_p)]


class Qkv4(ctypes.Structure):
    """Mirror of ra_qkv4 (device pointers)."""
    _fields_ = [("q4", ctypes.c_void_p), ("k4", ctypes.c_void_p), ("v4t", ctypes.c_void_p),
                ("sq", ctypes.c_void_p), ("sk", ctypes.c_void_p), ("sv", ctypes.c_void_p),
                ("vsum", ctypes.c_void_p)]


_lib = None
_P = ctypes.POINTER(Problem)
_V = ctypes.c_void_p
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "ra_seq_len": (ctypes.c_int, [_P]),
    "ra_seq_pad": (ctypes.c_int, [_P]),
    "ra_validate": (ctypes.c_int, [_P]),
    "ra_qkv4_bytes": (_SZ, [_P]),
    "ra_qkv4_bind": (ctypes.c_int, [_P, _V, _SZ, ctypes.POINTER(Qkv4)]),
    "ra_workspace_bytes": (_SZ, [_P, ctypes.c_int]),
    "ra_prepare": (ctypes.c_int, [_P, _V, _SZ, _V]),
    "ra_rotate_quantize_qkv": (ctypes.c_int, [_P, _V, _V, _V, ctypes.POINTER(Qkv4), _V, _SZ, _V]),
    "ra_int4_attention_fwd": (ctypes.c_int, [_P, ctypes.POINTER(Qkv4), _V, _V, _SZ, _V]),
    "ra_fp16_attention_fwd": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _SZ, _V]),
    "ra_check_device_error": (ctypes.c_int, [_V, _V]),
    "ra_host_staging_bytes": (_SZ, [_P, ctypes.c_int]),
    "ra_int4_attention_host": (ctypes.c_int, [_P, _V, _V, _V, _V, ctypes.c_int, _V, _SZ, _V]),
    "ra_host_chunks": (ctypes.c_int, [_P, ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_int]),
    "ra_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ra_last_error_detail": (ctypes.c_char_p, []),
    "ra_tables_floats": (_SZ, [_P]),
    "ra_build_tables_host": (ctypes.c_int, [_P, _V, _SZ]),
    "ra_debug_int4_tile": (ctypes.c_int, [_P, ctypes.POINTER(Qkv4), ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _V, _V, _V, _SZ, _V]),
    "ra_rotate_quantize_qkv_noalloc": (ctypes.c_int, [_P, _V, _V, _V, ctypes.POINTER(Qkv4), _V]),
    "ra_noalloc_check_device_error": (ctypes.c_int, [_V]),
    "ra_debug_set_wait_timeout_us": (None, [ctypes.c_uint32]),
    "ra_debug_timeout_probe": (ctypes.c_int, [_V, _SZ, _V]),
    "ra_measure_mma_i8": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _V, _SZ, _V]),
    "ra_debug_ex2": (ctypes.c_int, [_V, _V, ctypes.c_int, _V]),
}


def lib():
    """Load librotate_attn.so (built in-tree by ``build.build()``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RotateAttnError("load", RA_ERR_CUDA,
                                  f"{LIB_PATH} is missing; run int4_quantized_attention_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ra_status_string(status).decode()


def _check(call: str, status: int) -> None:
    if status != RA_OK:
        raise RotateAttnError(call, status, lib().ra_last_error_detail().decode())


def problem(cfg, rot: Optional[str] = None) -> Problem:
    """ra_problem from any object with B, H, d, F, Hh, W, n_text, split, theta, rot."""
    p = Problem()
    p.B, p.H, p.d = cfg.B, cfg.H, cfg.d
    p.F, p.Hh, p.W, p.n_text = cfg.F, cfg.Hh, cfg.W, cfg.n_text
    p.split = (ctypes.c_int * 3)(*cfg.split)
    p.theta = float(cfg.theta)
    p.rot = ROT[rot if rot is not None else cfg.rot]
    p.p_mode = P_MODE[getattr(cfg, "p_mode", "range")]
    p.v_rot = int(getattr(cfg, "v_rot", 0))
    blocks = getattr(cfg, "blocks", None)
    if blocks is not None:
        arr = (ctypes.c_double * len(blocks))(*blocks)
        p._keep = arr                      # the array lives as long as the struct
        p.blocks = ctypes.cast(arr, ctypes.c_void_p)
    return p


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


# ---------------------------------------------------------------- C entry points

def seq_len(p: Problem) -> int:
    return lib().ra_seq_len(ctypes.byref(p))


def seq_pad(p: Problem) -> int:
    return lib().ra_seq_pad(ctypes.byref(p))


def validate(p: Problem) -> int:
    return lib().ra_validate(ctypes.byref(p))


def qkv4_bytes(p: Problem) -> int:
    return lib().ra_qkv4_bytes(ctypes.byref(p))


def qkv4_bind(p: Problem, buf) -> Qkv4:
    out = Qkv4()
    _check("ra_qkv4_bind", lib().ra_qkv4_bind(ctypes.byref(p), _ptr(buf), buf.numel() * buf.element_size(),
                                              ctypes.byref(out)))
    return out


def workspace_bytes(p: Problem, with_fp16_path: bool = True) -> int:
    return lib().ra_workspace_bytes(ctypes.byref(p), int(with_fp16_path))


def prepare(p: Problem, workspace, stream=None) -> None:
    _check("ra_prepare", lib().ra_prepare(ctypes.byref(p), _ptr(workspace), workspace.numel(), _stream(stream)))


def rotate_quantize_qkv(p: Problem, q, k, v, out: Qkv4, workspace, stream=None) -> None:
    _check("ra_rotate_quantize_qkv",
           lib().ra_rotate_quantize_qkv(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(out),
                                        _ptr(workspace), workspace.numel(), _stream(stream)))


def int4_attention_fwd(p: Problem, qkv4: Qkv4, o, workspace, stream=None) -> None:
    _check("ra_int4_attention_fwd",
           lib().ra_int4_attention_fwd(ctypes.byref(p), ctypes.byref(qkv4), _ptr(o), _ptr(workspace),
                                       workspace.numel(), _stream(stream)))


def fp16_attention_fwd(p: Problem, q, k, v, o, workspace, stream=None) -> None:
    _check("ra_fp16_attention_fwd",
           lib().ra_fp16_attention_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(workspace),
                                       workspace.numel(), _stream(stream)))


def host_staging_bytes(p: Problem, heads_per_chunk: int = 0) -> int:
    return lib().ra_host_staging_bytes(ctypes.byref(p), heads_per_chunk)


def host_chunks(p: Problem, heads_per_chunk: int = 0) -> list:
    """Heads per chunk, in order, of ra_int4_attention_host's pipeline."""
    n = lib().ra_host_chunks(ctypes.byref(p), heads_per_chunk, None, 0)
    if n < 0:
        _check("ra_host_chunks", RA_ERR_INVALID_ARG)
    out = (ctypes.c_int * max(n, 1))()
    lib().ra_host_chunks(ctypes.byref(p), heads_per_chunk, out, n)
    return list(out[:n])


def int4_attention_host(p: Problem, q, k, v, o, staging, heads_per_chunk: int = 0, stream=None) -> None:
    """The INT4 path from host q, k, v to host o (CPU tensors, page-locked for
    overlap); blocks until o is written."""
    _check("ra_int4_attention_host",
           lib().ra_int4_attention_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), heads_per_chunk,
                                        _ptr(staging), staging.numel(), _stream(stream)))


def rotate_quantize_qkv_noalloc(p: Problem, q, k, v, out: Qkv4, stream=None) -> None:
    """The prologue with its scratch in the library's fixed device array."""
    _check("ra_rotate_quantize_qkv_noalloc",
           lib().ra_rotate_quantize_qkv_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(out),
                                                _stream(stream)))


def noalloc_check_device_error(stream=None) -> None:
    """Read and clear the error word of the allocation-free prologue's scratch."""
    _check("ra_noalloc_check_device_error", lib().ra_noalloc_check_device_error(_stream(stream)))


def check_device_error(workspace, stream=None) -> None:
    _check("ra_check_device_error", lib().ra_check_device_error(_ptr(workspace), _stream(stream)))


def build_tables_host(p: Problem):
    import numpy as np
    n = lib().ra_tables_floats(ctypes.byref(p))
    out = np.empty((n,), np.float32)
    _check("ra_build_tables_host",
           lib().ra_build_tables_host(ctypes.byref(p), out.ctypes.data_as(ctypes.c_void_p), n))
    return out.reshape(-1, 4)


def debug_int4_tile(p: Problem, qkv4: Qkv4, bh: int, q_tile: int, kv_tile: int, workspace, stream=None):
    """int32 S tile [128, 128] and int8 P codes [128, 128] of one (head, q tile, kv tile)."""
    import torch
    dev = workspace.device
    s_out = torch.zeros((128, 128), dtype=torch.int32, device=dev)
    p_out = torch.zeros((128, 128), dtype=torch.int8, device=dev)
    _check("ra_debug_int4_tile",
           lib().ra_debug_int4_tile(ctypes.byref(p), ctypes.byref(qkv4), bh, q_tile, kv_tile, _ptr(s_out),
                                    _ptr(p_out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return s_out, p_out


def debug_ex2(x, stream=None):
    """The attention kernel's 2^x (ex2.approx) of a device float32 tensor."""
    import torch
    y = torch.empty_like(x)
    _check("ra_debug_ex2", lib().ra_debug_ex2(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def debug_set_wait_timeout_us(microseconds: int) -> None:
    lib().ra_debug_set_wait_timeout_us(microseconds)


def debug_timeout_probe(workspace, stream=None) -> None:
    _check("ra_debug_timeout_probe",
           lib().ra_debug_timeout_probe(_ptr(workspace), workspace.numel(), _stream(stream)))


def measure_mma_i8(n: int, iters: int, ctas: int, workspace, stream=None) -> None:
    """Enqueue the INT8 tensor-core rate probe (ctas * iters * 4 * 2 * 128 * n * 32 ops)."""
    _check("ra_measure_mma_i8", lib().ra_measure_mma_i8(n, iters, ctas, _ptr(workspace), workspace.numel(),
                                                        _stream(stream)))


# ---------------------------------------------------------------- convenience

class RotateAttention:
    """Owns (through PyTorch) the workspace and the quantised-QKV buffer of one
    problem and calls the C entry points on the current stream."""

    def __init__(self, cfg, device="cuda", fp16_path: bool = True):
        import torch
        self.cfg = cfg
        self.p = problem(cfg)
        _check("ra_validate", validate(self.p))
        self.N = seq_len(self.p)
        self.N_pad = seq_pad(self.p)
        self.device = torch.device(device)
        self.workspace = torch.empty((workspace_bytes(self.p, fp16_path),), dtype=torch.uint8, device=self.device)
        self.qkv4_buf = torch.empty((qkv4_bytes(self.p),), dtype=torch.uint8, device=self.device)
        self.qkv4 = qkv4_bind(self.p, self.qkv4_buf)
        prepare(self.p, self.workspace)

    def rotate_quantize(self, q, k, v) -> Qkv4:
        rotate_quantize_qkv(self.p, q, k, v, self.qkv4, self.workspace)
        return self.qkv4

    def int4_attention(self, out=None):
        import torch
        if out is None:
            out = torch.empty((self.cfg.B, self.cfg.H, self.N, self.cfg.d), dtype=torch.float16, device=self.device)
        int4_attention_fwd(self.p, self.qkv4, out, self.workspace)
        return out

    def fp16_attention(self, q, k, v, out=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        fp16_attention_fwd(self.p, q, k, v, out, self.workspace)
        return out

    def forward(self, q, k, v, path: str = "int4", out=None):
        if path == "int4":
            self.rotate_quantize(q, k, v)
            return self.int4_attention(out)
        if path == "fp16":
            return self.fp16_attention(q, k, v, out)
        raise ValueError(path)

    def forward_host(self, q, k, v, out, heads_per_chunk: int = 0):
        """INT4 path on host tensors (q, k, v, out on the CPU, page-locked for
        overlap): copies, kernels and copies back pipelined over head chunks
        by the library.  Returns once out is written."""
        import torch
        need = host_staging_bytes(self.p, heads_per_chunk)
        if getattr(self, "_staging", None) is None or self._staging.numel() < need:
            self._staging = torch.empty((need,), dtype=torch.uint8, device=self.device)
        int4_attention_host(self.p, q, k, v, out, self._staging, heads_per_chunk)
        return out

    def check(self) -> None:
        check_device_error(self.workspace)

    def unpack(self):
        """Host copies of the quantised tensors (int8 codes, unpacked), for tests."""
        import numpy as np
        import torch
        BH, Np = self.cfg.B * self.cfg.H, self.N_pad
        torch.cuda.synchronize()
        buf = self.qkv4_buf.cpu().numpy()
        base = self.qkv4_buf.data_ptr()

        def view(ptr, nbytes, dtype):
            off = ptr - base
            return buf[off:off + nbytes].view(dtype)

        packed = BH * Np * 64
        q4 = view(self.qkv4.q4, packed, np.uint8).reshape(BH, Np, 64)
        k4 = view(self.qkv4.k4, packed, np.uint8).reshape(BH, Np, 64)
        v4t = view(self.qkv4.v4t, packed, np.uint8).reshape(BH, Np // 128, 128, 64)
        sq = view(self.qkv4.sq, BH * (Np // 64) * 4, np.float32).reshape(BH, Np // 64)
        sk = view(self.qkv4.sk, BH * (Np // 64) * 4, np.float32).reshape(BH, Np // 64)
        sv = view(self.qkv4.sv, BH * 128 * 4, np.float32).reshape(BH, 128)
        vsum = view(self.qkv4.vsum, BH * (Np // 64) * 128 * 4, np.int32).reshape(BH, Np // 64, 128)
        return dict(qc=unpack_nibbles(q4), kc=unpack_nibbles(k4),
                    vc=np.ascontiguousarray(unpack_nibbles(v4t).transpose(0, 1, 3, 2).reshape(BH, Np, 128)),
                    qs=sq, ks=sk, sv=sv, colsum=vsum)


def unpack_nibbles(packed):
    """uint8 [..., n] with two's-complement nibbles -> int8 [..., 2n], low nibble first."""
    import numpy as np
    lo = (packed & 0x0F).astype(np.int8)
    hi = (packed >> 4).astype(np.int8)
    lo = np.where(lo > 7, lo - 16, lo).astype(np.int8)
    hi = np.where(hi > 7, hi - 16, hi).astype(np.int8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out
