"""Python front of the CPU oracle (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this module.  It loads ``liboracle.so`` (plain C, built from
``rotate_attn_oracle.c`` by ``build_oracle()``) and marshals numpy arrays;
all arithmetic is in the C file.  It never imports the CUDA package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rotate_attn_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
ROT = {"none": 0, "interleaved": 1, "half": 2, "full": 3, "blocks_interleaved": 4, "blocks_half": 5}


def compile_oracle(src: str, out: str) -> None:
    """gcc, IEEE fp32 with no FMA contraction, OpenMP over independent rows."""
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", out + ".tmp", src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)


def build_oracle(force: bool = False) -> str:
    """Build liboracle.so next to its source (or return RA_ORACLE_LIB if set:
    the mutation test points the pins at deliberately broken copies)."""
    override = os.environ.get("RA_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_oracle(SRC, LIB)
    return LIB


class _Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("F", ctypes.c_int), ("Hh", ctypes.c_int), ("W", ctypes.c_int),
                ("n_text", ctypes.c_int), ("split", ctypes.c_int * 3),
                ("theta", ctypes.c_double), ("rot", ctypes.c_int), ("v_rot", ctypes.c_int),
                ("blocks", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_oracle())
        _lib.orc_p_code.restype = ctypes.c_int
        _lib.orc_p_code.argtypes = [ctypes.c_float]
        _lib.orc_p_code_sym.restype = ctypes.c_int
        _lib.orc_p_code_sym.argtypes = [ctypes.c_float]
        _lib.orc_p_weight.restype = ctypes.c_int
        _lib.orc_p_weight.argtypes = [ctypes.c_float, ctypes.c_int]
        _lib.orc_p_weight_amb.restype = ctypes.c_int
        _lib.orc_p_weight_amb.argtypes = [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
        _lib.orc_rope_angle.restype = ctypes.c_double
        _lib.orc_seq_len.restype = ctypes.c_int
        _lib.orc_seq_pad.restype = ctypes.c_int
    return _lib


def problem(cfg, rot: Optional[str] = None) -> _Problem:
    """Oracle problem struct from a synth.Config-like object."""
    p = _Problem()
    p.B, p.H, p.d = cfg.B, cfg.H, cfg.d
    p.F, p.Hh, p.W, p.n_text = cfg.F, cfg.Hh, cfg.W, cfg.n_text
    p.split = (ctypes.c_int * 3)(*cfg.split)
    p.theta = float(cfg.theta)
    p.rot = ROT[rot if rot is not None else cfg.rot]
    p.v_rot = int(getattr(cfg, "v_rot", 0))
    blocks = getattr(cfg, "blocks", None)
    if blocks is not None:
        arr = (ctypes.c_double * len(blocks))(*blocks)
        p._keep = arr                      # the array lives as long as the struct
        p.blocks = ctypes.cast(arr, ctypes.c_void_p)
    return p


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def n_pad(cfg) -> int:
    return (cfg.N + 127) // 128 * 128


def token_pos(cfg, n: int):
    pos = (ctypes.c_int * 3)()
    lib().orc_token_pos(ctypes.byref(problem(cfg)), n, pos)
    return tuple(pos)


def rope_coef(cfg, s: int, pos: int, j: int):
    """(cos, sin, alpha, beta) fp32 coefficients for segment s, position, pair j."""
    c, sn, al, be = (ctypes.c_float() for _ in range(4))
    lib().orc_rope_coef(ctypes.byref(problem(cfg)), s, pos, j,
                        ctypes.byref(c), ctypes.byref(sn), ctypes.byref(al), ctypes.byref(be))
    return np.float32(c.value), np.float32(sn.value), np.float32(al.value), np.float32(be.value)


def rope_angle(cfg, s: int, pos: int, j: int) -> float:
    return lib().orc_rope_angle(ctypes.byref(problem(cfg)), s, pos, j)


def p_code(P: float) -> int:
    return lib().orc_p_code(ctypes.c_float(P))


def p_code_sym(P: float) -> int:
    return lib().orc_p_code_sym(ctypes.c_float(P))


def p_weight(x: float, levels: int = 15) -> int:
    """rne(levels * 2^x) for the fp32 exponent x (the quantised path's P weight)."""
    return lib().orc_p_weight(ctypes.c_float(x), levels)


def p_weight_amb(x: float, levels: int = 15):
    """(weight, ambiguous?) for the fp32 exponent x."""
    amb = ctypes.c_int(0)
    w = lib().orc_p_weight_amb(ctypes.c_float(x), levels, ctypes.byref(amb))
    return w, bool(amb.value)


def _quant_mode(cfg, quant_p) -> int:
    """0: exact P; 1: range-optimised P code; 2: symmetric P code."""
    if not quant_p:
        return 0
    return 2 if getattr(cfg, "p_mode", "range") == "symmetric" else 1


def rotate_head(cfg, x: np.ndarray, rot: Optional[str] = None) -> np.ndarray:
    """fp32 rows after RoPE + rotation; x: fp16 [N, d]."""
    x = np.ascontiguousarray(x, np.float16)
    z = np.empty(x.shape, np.float32)
    lib().orc_rotate_head(ctypes.byref(problem(cfg, rot)), _ptr(x), _ptr(z))
    return z


def rope_fp16_head(cfg, x: np.ndarray) -> np.ndarray:
    """fp16 rows after RoPE only (the FP16 path's position encoding)."""
    x = np.ascontiguousarray(x, np.float16)
    y = np.empty(x.shape, np.float16)
    lib().orc_rope_fp16_head(ctypes.byref(problem(cfg, "none")), _ptr(x), _ptr(y))
    return y


def quantize_qk_head(cfg, x: np.ndarray, rot: Optional[str] = None):
    """INT4 codes [N_pad, d] (int8 values) and 64-token block scales [N_pad/64]."""
    x = np.ascontiguousarray(x, np.float16)
    Np = n_pad(cfg)
    codes = np.empty((Np, cfg.d), np.int8)
    scales = np.empty((Np // 64,), np.float32)
    lib().orc_quantize_qk_head(ctypes.byref(problem(cfg, rot)), _ptr(x), _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_v_head(cfg, v: np.ndarray):
    """V codes [N_pad, d], channel scales [d], 64-block column sums [N_pad/64, d]."""
    v = np.ascontiguousarray(v, np.float16)
    Np = n_pad(cfg)
    codes = np.empty((Np, cfg.d), np.int8)
    sv = np.empty((cfg.d,), np.float32)
    colsum = np.empty((Np // 64, cfg.d), np.int32)
    lib().orc_quantize_v_head(ctypes.byref(problem(cfg)), _ptr(v), _ptr(codes), _ptr(sv), _ptr(colsum))
    return codes, sv, colsum


def quantize_head(cfg, q, k, v, rot: Optional[str] = None):
    """All prologue outputs of one head, as a dict."""
    qc, qs = quantize_qk_head(cfg, q, rot)
    kc, ks = quantize_qk_head(cfg, k, rot)
    vc, sv, cs = quantize_v_head(cfg, v)
    return dict(qc=qc, qs=qs, kc=kc, ks=ks, vc=vc, sv=sv, colsum=cs)


MAX_AMB = 8     # ambiguous keys recorded per row


def attention_rows(cfg, qz: dict, rows=None, tile: int = 128, quant_p: bool = True,
                   want64: bool = False, ambiguous: bool = False):
    """INT4 attention output rows of one head from the prologue outputs `qz`.
    With ambiguous=True also returns, per row, the number of keys whose P
    code is ambiguous (either rounding is a correct fp32 decision) and the
    first MAX_AMB of them."""
    if quant_p and tile % 64:
        raise ValueError("the zero-point column sums need tiles that are whole 64-token blocks")
    rows = np.arange(cfg.N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    out = np.empty((len(rows), cfg.d), np.float16)
    out64 = np.empty((len(rows), cfg.d), np.float64) if want64 else None
    cnt = np.zeros((len(rows),), np.int32) if ambiguous else None
    keys = np.full((len(rows), MAX_AMB), -1, np.int32) if ambiguous else None
    lib().orc_attention_rows(ctypes.byref(problem(cfg)), _ptr(rows), len(rows), tile, _quant_mode(cfg, quant_p),
                             _ptr(qz["qc"]), _ptr(qz["qs"]), _ptr(qz["kc"]), _ptr(qz["ks"]),
                             _ptr(qz["vc"]), _ptr(qz["sv"]), _ptr(qz["colsum"]), _ptr(out),
                             _ptr(out64) if want64 else None, _ptr(cnt) if ambiguous else None,
                             _ptr(keys) if ambiguous else None, MAX_AMB)
    res = (out, out64) if want64 else out
    return (res, cnt, keys) if ambiguous else res


def attention_row_debug(cfg, qz: dict, i: int, tile_index: int, tile: int = 128, with_ambiguous: bool = False):
    """S (int32) and P codes (int8; -128 past N) of one row for one KV tile;
    with_ambiguous=True adds a mask of the tile's keys whose P code is
    ambiguous (either neighbouring code is a correct fp32 decision)."""
    S = np.zeros((tile,), np.int32)
    P = np.zeros((tile,), np.int8)
    o = np.empty((cfg.d,), np.float16)
    amb = np.full((4096,), -1, np.int32)
    cnt = ctypes.c_int32(0)
    lib().orc_attention_row(ctypes.byref(problem(cfg)), i, tile, _quant_mode(cfg, True),
                            _ptr(qz["qc"]), _ptr(qz["qs"]), _ptr(qz["kc"]), _ptr(qz["ks"]),
                            _ptr(qz["vc"]), _ptr(qz["sv"]), _ptr(qz["colsum"]), _ptr(o), None,
                            tile_index, _ptr(S), _ptr(P), _ptr(amb), len(amb), ctypes.byref(cnt), None, 0)
    if not with_ambiguous:
        return S, P
    keys = amb[:min(cnt.value, len(amb))]
    in_tile = keys[(keys >= tile_index * tile) & (keys < tile_index * tile + tile)] - tile_index * tile
    mask = np.zeros((tile,), bool)
    mask[in_tile] = True
    return S, P, mask


def attention_row_flipped(cfg, qz: dict, i: int, flip, tile: int = 128):
    """Float64 output row i with the ambiguous keys in `flip` decided the
    other way (one of the other correct results)."""
    flip = np.ascontiguousarray(flip, np.int32)
    o = np.empty((cfg.d,), np.float16)
    o64 = np.empty((cfg.d,), np.float64)
    lib().orc_attention_row(ctypes.byref(problem(cfg)), i, tile, _quant_mode(cfg, True),
                            _ptr(qz["qc"]), _ptr(qz["qs"]), _ptr(qz["kc"]), _ptr(qz["ks"]),
                            _ptr(qz["vc"]), _ptr(qz["sv"]), _ptr(qz["colsum"]), _ptr(o), _ptr(o64),
                            -1, None, None, None, 0, None, _ptr(flip) if len(flip) else None, len(flip))
    return o64


def softmax_attention_rows(cfg, q: np.ndarray, k: np.ndarray, v: np.ndarray, rows=None) -> np.ndarray:
    """Float64 softmax attention (1/sqrt d) of one head on given rows."""
    rows = np.arange(cfg.N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty((len(rows), cfg.d), np.float64)
    lib().orc_softmax_attention_rows(ctypes.byref(problem(cfg)), _ptr(rows), len(rows),
                                     _ptr(q), _ptr(k), _ptr(v), _ptr(out))
    return out


def exact_attention_rows(cfg, q, k, v, rows=None) -> np.ndarray:
    """Unquantised diagnostic: RoPE + rotation in fp32, then float64 attention."""
    zq = rotate_head(cfg, q)
    zk = rotate_head(cfg, k)
    return softmax_attention_rows(cfg, zq, zk, v.astype(np.float64), rows)


def fp16_attention_rows(cfg, q, k, v, rows=None) -> np.ndarray:
    """FP16 path oracle: RoPE rounded to fp16, then float64 attention."""
    return softmax_attention_rows(cfg, rope_fp16_head(cfg, q), rope_fp16_head(cfg, k),
                                  v.astype(np.float64), rows)
