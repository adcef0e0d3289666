"""CSA2 decode oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow CPU statement of every step of the CSA2 sparse-attention decode
path (C in ``csa2_oracle.c``, driven from numpy through ctypes).  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package; the product library never does, and this package
never imports the product.  It shares no code with the CUDA path.

Every function cites the passage it follows in the C source.  Pins (tests
under ``tests/test_oracle_*.py``) tie it to closed forms, brute force and
library routines rather than to itself.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

LATENT, GROUP, IDX_DIM, IDX_HEADS = 512, 16, 128, 32
BLOCK, MAX_BLOCKS, POOL, TOPK, SWA = 8, 2048, 16384, 512, 128
CODE_BYTES, SCALE_BYTES = LATENT // 2, LATENT // GROUP


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -ffp-contract=off, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            P = C.c_void_p
            for name, res, args in [
                ("orc_e2m1_decode", C.c_double, [C.c_uint8]),
                ("orc_e4m3_decode", C.c_double, [C.c_uint8]),
                ("orc_e2m1_encode", C.c_uint8, [C.c_float]),
                ("orc_e4m3_encode", C.c_uint8, [C.c_float]),
                ("orc_e2m1_encode_n", None, [P, C.c_long, P]),
                ("orc_e4m3_encode_n", None, [P, C.c_long, P]),
                ("orc_e2m1_decode_n", None, [P, C.c_long, P]),
                ("orc_e4m3_decode_n", None, [P, C.c_long, P]),
                ("orc_swa_quant_n", None, [P, C.c_long, P, P]),
                ("orc_compress", None, [C.c_int, P, P, C.c_int, P]),
                ("orc_pack_latent", None, [P, P, P]),
                ("orc_unpack_latent", None, [P, P, P]),
                ("orc_block_summary", None, [P, C.c_int, P]),
                ("orc_build_entries", None, [C.c_int, C.c_int, C.c_int, P, P, P, P, P, P]),
                ("orc_build_summaries", None, [P, C.c_int, P]),
                ("orc_index_score_f64", C.c_double, [P, P, P]),
                ("orc_score_rows", None, [P, P, P, C.c_int, P, P]),
                ("orc_topk", C.c_int, [P, P, C.c_int, C.c_int, P]),
                ("orc_index_flat", C.c_int, [P, P, P, C.c_int, P]),
                ("orc_expand_pool", C.c_int, [P, C.c_int, C.c_int, P]),
                ("orc_index_pool", C.c_int, [P, P, P, P, C.c_int, P]),
                ("orc_index_full", C.c_int, [P, P, P, P, C.c_int, P, P, P]),
                ("orc_attend", None, [C.c_int, P, C.c_int, P, P, C.c_int, P, P, C.c_double, P]),
                ("orc_attend_lse", None, [C.c_int, P, C.c_int, P, P, C.c_int, P, P, C.c_double, P, P]),
                ("orc_lse_combine", None, [C.c_int, C.c_int, P, P, P]),
            ]:
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


# ---------------------------------------------------------------- formats
def e2m1_encode(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(x), x.size, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(x), x.size, _p(out))
    return out


def e2m1_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e2m1_decode_n(_p(c), c.size, _p(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_n(_p(c), c.size, _p(out))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = _c(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- append
def compress(m: int, x, g) -> np.ndarray:
    """x: [m, dim] float32, g: [m] -> [dim] float32."""
    x = _c(x, np.float32)
    g = _c(g, np.float32)
    out = np.empty(x.shape[-1], np.float32)
    lib().orc_compress(m, _p(x), _p(g), x.shape[-1], _p(out))
    return out


def pack_latent(e):
    e = _c(e, np.float32)
    assert e.shape == (LATENT,)
    codes = np.empty(CODE_BYTES, np.uint8)
    scales = np.empty(SCALE_BYTES, np.uint8)
    lib().orc_pack_latent(_p(e), _p(codes), _p(scales))
    return codes, scales


def unpack_latent(codes, scales) -> np.ndarray:
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    out = np.empty(LATENT, np.float64)
    lib().orc_unpack_latent(_p(codes), _p(scales), _p(out))
    return out


def block_summary(keys8) -> np.ndarray:
    keys8 = _c(keys8, np.uint8)
    out = np.empty(IDX_DIM, np.uint8)
    lib().orc_block_summary(_p(keys8), keys8.shape[0], _p(out))
    return out


def swa_quant(x):
    """x: [n, 512] float32 -> (codes [n, 512] u8, scale [n] f32)."""
    x = _c(x, np.float32).reshape(-1, LATENT)
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[0], np.float32)
    lib().orc_swa_quant_n(_p(x), x.shape[0], _p(codes), _p(scale))
    return codes, scale


def build_entries(m: int, tok_lat, tok_key, tok_gate, e_begin: int = 0, with_latent: bool = True):
    """Entries [e_begin, e_begin + n) from tokens [m*e_begin, ...): the token
    arrays hold exactly those tokens.  Returns (codes, scales, keys8)."""
    tok_key = _c(tok_key, np.float32)
    tok_gate = _c(tok_gate, np.float32)
    n = tok_key.shape[0] // m
    keys8 = np.empty((n, IDX_DIM), np.uint8)
    if with_latent:
        tok_lat = _c(tok_lat, np.float32)
        codes = np.empty((n, CODE_BYTES), np.uint8)
        scales = np.empty((n, SCALE_BYTES), np.uint8)
        lib().orc_build_entries(m, e_begin, e_begin + n, _p(tok_lat), _p(tok_key), _p(tok_gate),
                                _p(codes), _p(scales), _p(keys8))
        return codes, scales, keys8
    dummy = np.zeros(1, np.float32)
    lib().orc_build_entries(m, e_begin, e_begin + n, _p(dummy), _p(tok_key), _p(tok_gate),
                            None, None, _p(keys8))
    return None, None, keys8


def build_summaries(keys8) -> np.ndarray:
    keys8 = _c(keys8, np.uint8)
    n = keys8.shape[0]
    nb = (n + BLOCK - 1) // BLOCK
    out = np.empty((nb, IDX_DIM), np.uint8)
    lib().orc_build_summaries(_p(keys8), n, _p(out))
    return out


def swa_window(tok_lat_tail, n_tok: int):
    """SWA ring of a request that has seen n_tok tokens; tok_lat_tail holds
    its last min(n_tok, 128) raw tokens.  Returns (codes [128,512],
    scale [128], valid) with token pos in slot pos % 128."""
    nv = min(n_tok, SWA)
    tail = _c(tok_lat_tail, np.float32).reshape(-1, LATENT)
    assert tail.shape[0] == nv
    codes = np.zeros((SWA, LATENT), np.uint8)
    scale = np.zeros(SWA, np.float32)
    if nv:
        c, s = swa_quant(tail)
        slots = (np.arange(n_tok - nv, n_tok) % SWA)
        codes[slots] = c
        scale[slots] = s
    return codes, scale, nv


# ---------------------------------------------------------------- indexer
def score_f64(q_bits, w, rows8) -> np.ndarray:
    q_bits, w, rows8 = _c(q_bits, np.uint16), _c(w, np.float32), _c(rows8, np.uint8)
    n = rows8.shape[0]
    s64 = np.empty(n, np.float64)
    lib().orc_score_rows(_p(q_bits), _p(w), _p(rows8), n, None, _p(s64))
    return s64


def score_f32(q_bits, w, rows8) -> np.ndarray:
    return score_f64(q_bits, w, rows8).astype(np.float32)


def topk(scores, k: int, ids=None) -> np.ndarray:
    s = _c(scores, np.float32)
    out = np.empty(k, np.int32)
    if ids is None:
        lib().orc_topk(_p(s), None, s.size, k, _p(out))
    else:
        ids = _c(ids, np.int32)
        lib().orc_topk(_p(s), _p(ids), s.size, k, _p(out))
    return out


def index_flat(q_bits, w, keys8) -> np.ndarray:
    q_bits, w, keys8 = _c(q_bits, np.uint16), _c(w, np.float32), _c(keys8, np.uint8)
    out = np.empty(TOPK, np.int32)
    lib().orc_index_flat(_p(q_bits), _p(w), _p(keys8), keys8.shape[0], _p(out))
    return out


def expand_pool(blocks, n_entries: int):
    blocks = _c(blocks, np.int32)
    pool = np.empty(POOL, np.int32)
    n = lib().orc_expand_pool(_p(blocks), blocks.size, n_entries, _p(pool))
    return pool, n


def index_pool(q_bits, w, keys8, pool, pool_len: int) -> np.ndarray:
    q_bits, w, keys8 = _c(q_bits, np.uint16), _c(w, np.float32), _c(keys8, np.uint8)
    pool = _c(pool, np.int32)
    out = np.empty(TOPK, np.int32)
    lib().orc_index_pool(_p(q_bits), _p(w), _p(keys8), _p(pool), pool_len, _p(out))
    return out


def index_full(q_bits, w, keys8, summ):
    """Returns (blocks [2048], pool [16384], pool_len, topk [512])."""
    q_bits, w = _c(q_bits, np.uint16), _c(w, np.float32)
    keys8, summ = _c(keys8, np.uint8), _c(summ, np.uint8)
    blocks = np.empty(MAX_BLOCKS, np.int32)
    pool = np.empty(POOL, np.int32)
    out = np.empty(TOPK, np.int32)
    n = lib().orc_index_full(_p(q_bits), _p(w), _p(keys8), _p(summ), keys8.shape[0],
                             _p(blocks), _p(pool), _p(out))
    return blocks, pool, n, out


# ---------------------------------------------------------------- attention
def attend(q_bits, codes_sel, scales_sel, swa_codes, swa_scale, scale: float) -> np.ndarray:
    """q_bits [H, 512] bf16 bits; codes_sel [n, 256], scales_sel [n, 32] of the
    selected FP4 entries; swa_codes [n_swa, 512], swa_scale [n_swa] of the
    valid window tokens.  Returns fp64 [H, 512]."""
    q_bits = _c(q_bits, np.uint16)
    H = q_bits.shape[0]
    codes_sel = _c(codes_sel, np.uint8).reshape(-1, CODE_BYTES)
    scales_sel = _c(scales_sel, np.uint8).reshape(-1, SCALE_BYTES)
    swa_codes = _c(swa_codes, np.uint8).reshape(-1, LATENT)
    swa_scale = _c(swa_scale, np.float32).reshape(-1)
    out = np.empty((H, LATENT), np.float64)
    lib().orc_attend(H, _p(q_bits), codes_sel.shape[0], _p(codes_sel), _p(scales_sel),
                     swa_codes.shape[0], _p(swa_codes), _p(swa_scale), float(scale), _p(out))
    return out


def attend_lse(q_bits, codes_sel, scales_sel, swa_codes, swa_scale, scale: float):
    """attend() plus, per head, ln sum_j exp(scale * q_h . v_j) (-inf when
    there are no keys).  Returns (fp64 [H, 512], fp64 [H])."""
    q_bits = _c(q_bits, np.uint16)
    H = q_bits.shape[0]
    codes_sel = _c(codes_sel, np.uint8).reshape(-1, CODE_BYTES)
    scales_sel = _c(scales_sel, np.uint8).reshape(-1, SCALE_BYTES)
    swa_codes = _c(swa_codes, np.uint8).reshape(-1, LATENT)
    swa_scale = _c(swa_scale, np.float32).reshape(-1)
    out = np.empty((H, LATENT), np.float64)
    lse = np.empty(H, np.float64)
    lib().orc_attend_lse(H, _p(q_bits), codes_sel.shape[0], _p(codes_sel), _p(scales_sel),
                         swa_codes.shape[0], _p(swa_codes), _p(swa_scale), float(scale), _p(out), _p(lse))
    return out, lse


def lse_combine(o_parts, lse_parts) -> np.ndarray:
    """Merge of attention results over disjoint key sets: o_parts [P, rows,
    512], lse_parts [P, rows] -> [rows, 512] fp64."""
    o_parts = _c(o_parts, np.float64)
    lse_parts = _c(lse_parts, np.float64)
    P, rows = lse_parts.shape
    assert o_parts.shape == (P, rows, LATENT)
    out = np.empty((rows, LATENT), np.float64)
    lib().orc_lse_combine(P, rows, _p(o_parts), _p(lse_parts), _p(out))
    return out
