"""CPU oracle for the MTP draft-head hot path -- TEST INFRASTRUCTURE ONLY.

A plain C library (``oracle/*.c``, fp64 accumulation, scalar loops) wrapped here with
ctypes for numpy arrays. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the CUDA library never does, and
the two share no code. bf16 arrays are passed as ``uint16`` bit patterns.

Each wrapped function names the C function that implements it; the C sources carry
the citations (the MTP head pages: spark_model/layers/mtp_head.rs,
metrale_model_layers/layers/mtp_head/new.rs, metrale_model_arch/glm5next_mtp_head/
init.rs, metrale_model_arch/deepseek_v4_mtp.rs) and the readings taken where the
pages are silent.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = ["formats.c", "quant.c", "draft.c", "prefill.c", "attn.c"]
LIB_PATH = os.path.join(_HERE, "liborc.so")

FLAG_BAD_TOKEN = 1
FLAG_EMPTY_MASK = 2
FLAG_BAD_SLOT = 4

FMT_BF16, FMT_FP8_ROW, FMT_NVFP4 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction, OpenMP)."""
    srcs = [os.path.join(_HERE, s) for s in _SRCS] + [os.path.join(_HERE, "oracle.h")]
    if not force and os.path.exists(LIB_PATH):
        so_t = os.path.getmtime(LIB_PATH)
        if all(os.path.getmtime(s) <= so_t for s in srcs):
            return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp]
    cmd += [os.path.join(_HERE, s) for s in _SRCS] + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


_lib = None

_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int32


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB_PATH)
        sig = {
            "orc_e4m3_value": (C.c_double, [C.c_uint8]),
            "orc_e2m1_value": (C.c_double, [C.c_uint8]),
            "orc_e4m3_encode": (C.c_uint8, [C.c_double]),
            "orc_e2m1_encode": (C.c_uint8, [C.c_double]),
            "orc_e4m3_encode_vec": (None, [_p, _i64, _p]),
            "orc_e2m1_encode_vec": (None, [_p, _i64, _p]),
            "orc_f64_to_bf16_vec": (None, [_p, _i64, _p]),
            "orc_quantize_fp8_rows": (None, [_p, _i64, _i64, _p, _p]),
            "orc_quantize_nvfp4": (None, [_p, _i64, _i64, _p, _p, _p]),
            "orc_dequant_row": (None, [_i32, _p, _p, _p, C.c_float, _i64, _i64, _p]),
            "orc_rmsnorm_row": (None, [_p, _p, _i64, C.c_double, _p]),
            "orc_combine": (_i32, [_p, _i64, _p, _p, _i32, _i32, _p, _p, C.c_double,
                                   _p, _p, _p]),
            "orc_lm_head_argmax": (_i32, [_i32, _p, _p, _p, C.c_float, _i64, _i64, _p,
                                          _i32, _p, _i64, _i64, _p, _p, _p]),
            "orc_argmax_masked": (_i32, [_p, _i64, _p, _i64, _p, _p]),
            "orc_top1_logprob": (C.c_double, [_p, _i64, _p, _i64]),
            "orc_rope_neox": (None, [_p, _i32, C.c_double, C.c_double, _p]),
            "orc_slot": (_i64, [_p, _i64, _i32, _i64, _i64]),
            "orc_kv_encode": (None, [_p, _i64, C.c_float, _p]),
            "orc_prefill_rows": (_i32, [_p, _i64, _p, _p, _i32, _p, _p, C.c_double, _p,
                                        _p, _p, _i32, _i32, C.c_double, _p, _i64, _p,
                                        _i64, _i32, _i64, C.c_float, C.c_float, _p,
                                        _i64, _p, _p, _p, _p, _p, _p]),
            "orc_rmsnorm_row_mode": (None, [_p, _p, _i64, C.c_double, _i32, _p]),
            "orc_combine_mode": (_i32, [_p, _i64, _p, _p, _i32, _i32, _p, _p, C.c_double, _i32,
                                        _p, _p, _p]),
            "orc_prefill_rows_ext": (_i32, [_p, _i64, _p, _p, _i32, _p, _p, C.c_double, _p,
                                            _p, _p, _i32, _i32, C.c_double, _p, _i64, _p,
                                            _i64, _i32, _i64, C.c_float, C.c_float, _i32, _p,
                                            _p, _p, _i64, _p, _p, _p, _p, _p, _p]),
            "orc_paged_decode_attn": (_i32, [_p, _i32, _i32, _i32, _p, _p, _p, _i64, _i32,
                                             _i64, _i64, C.c_double, C.c_double, C.c_double,
                                             _p]),
            "orc_num_threads": (_i32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---- formats (formats.c) -------------------------------------------------------

def e4m3_value(codes) -> np.ndarray:
    table = np.array([lib().orc_e4m3_value(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e2m1_value(codes) -> np.ndarray:
    table = np.array([lib().orc_e2m1_value(c) for c in range(16)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8) & 0xF]


def e4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_vec(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_encode(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_vec(_ptr(v), v.size, _ptr(out))
    return out


def bf16_to_f64(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_f64_to_bf16_vec(_ptr(v), v.size, _ptr(out))
    return out


# ---- quantizers (quant.c) ------------------------------------------------------

def quantize_fp8(w):
    w = _c(w, np.uint16)
    n, k = w.shape
    codes = np.empty((n, k), dtype=np.uint8)
    scale = np.empty((n,), dtype=np.float32)
    lib().orc_quantize_fp8_rows(_ptr(w), n, k, _ptr(codes), _ptr(scale))
    return codes, scale


def quantize_nvfp4(w):
    w = _c(w, np.uint16)
    n, k = w.shape
    assert k % 16 == 0
    codes = np.empty((n, k // 2), dtype=np.uint8)
    bscale = np.empty((n, k // 16), dtype=np.uint8)
    g = np.empty((1,), dtype=np.float32)
    lib().orc_quantize_nvfp4(_ptr(w), n, k, _ptr(codes), _ptr(bscale), _ptr(g))
    return codes, bscale, float(g[0])


def dequant(fmt, data, k, row_scale=None, block_scale=None, global_scale=0.0, rows=None):
    data = np.ascontiguousarray(data)
    n = data.shape[0]
    rows = range(n) if rows is None else rows
    rs = None if row_scale is None else _c(row_scale, np.float32)
    bs = None if block_scale is None else _c(block_scale, np.uint8)
    out = np.empty((len(rows), k), dtype=np.float64)
    for i, r in enumerate(rows):
        lib().orc_dequant_row(fmt, _ptr(data), _ptr(rs), _ptr(bs), float(global_scale), k,
                              int(r), _ptr(out[i]))
    return out


# ---- draft step (draft.c) ------------------------------------------------------

def rmsnorm(x, w, eps, norm_mode=0):
    """orc_rmsnorm_row_mode: weights w (norm_mode 0) or 1 + w (norm_mode 1)."""
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    y = np.empty_like(x)
    lib().orc_rmsnorm_row_mode(_ptr(x), _ptr(w), x.size, float(eps), int(norm_mode), _ptr(y))
    return y


def combine(embed, tokens, hidden, w_norm_embed, w_norm_hidden, eps, fc, norm_mode=0):
    embed = _c(embed, np.uint16)
    tokens = _c(tokens, np.int32)
    hidden = _c(hidden, np.uint16)
    M, h = hidden.shape
    concat = np.empty((M, 2 * h), dtype=np.uint16)
    y = np.empty((M, h), dtype=np.uint16)
    flags = lib().orc_combine_mode(_ptr(embed), embed.shape[0], _ptr(tokens), _ptr(hidden), M, h,
                                   _ptr(_c(w_norm_embed, np.uint16)),
                                   _ptr(_c(w_norm_hidden, np.uint16)), float(eps), int(norm_mode),
                                   _ptr(_c(fc, np.uint16)), _ptr(concat), _ptr(y))
    return y, concat, int(flags)


def lm_head_argmax(fmt, data, k, x, n_eff=None, row_scale=None, block_scale=None,
                   global_scale=0.0, mask=None, mask_words=0, mask_stride_words=0,
                   want_logits=True):
    """Returns (logits [M, n_eff] float64 or None, idx [M] int32, val [M] float64, flags)."""
    data = np.ascontiguousarray(data)
    x = _c(x, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    M = x.shape[0]
    n_eff = data.shape[0] if n_eff is None else int(n_eff)
    rs = None if row_scale is None else _c(row_scale, np.float32)
    bs = None if block_scale is None else _c(block_scale, np.uint8)
    mk = None if mask is None else _c(mask, np.int32)
    logits = np.empty((M, n_eff), dtype=np.float64) if want_logits else None
    idx = np.empty((M,), dtype=np.int32)
    val = np.empty((M,), dtype=np.float64)
    flags = lib().orc_lm_head_argmax(fmt, _ptr(data), _ptr(rs), _ptr(bs), float(global_scale),
                                     n_eff, k, _ptr(x), M, _ptr(mk), int(mask_words),
                                     int(mask_stride_words), _ptr(logits), _ptr(idx),
                                     _ptr(val))
    return logits, idx, val, int(flags)


def argmax_masked(logits, mask=None, mask_words=0):
    logits = _c(logits, np.float64)
    mk = None if mask is None else _c(mask, np.int32)
    idx = np.empty((1,), dtype=np.int32)
    val = np.empty((1,), dtype=np.float64)
    flags = lib().orc_argmax_masked(_ptr(logits), logits.size, _ptr(mk), int(mask_words),
                                    _ptr(idx), _ptr(val))
    return int(idx[0]), float(val[0]), int(flags)


def top1_logprob(logits, mask=None, mask_words=0) -> float:
    """Log-softmax at the argmax over the allowed tokens of one logit row."""
    logits = _c(logits, np.float64)
    mk = None if mask is None else _c(mask, np.int32)
    return float(lib().orc_top1_logprob(_ptr(logits), logits.size, _ptr(mk), int(mask_words)))


# ---- prefill (prefill.c) -------------------------------------------------------

def rope_neox(k, pos, base):
    k = _c(k, np.float64)
    out = np.empty_like(k)
    lib().orc_rope_neox(_ptr(k), k.size, float(pos), float(base), _ptr(out))
    return out


def slot(block_table, block_size, num_blocks, p):
    bt = _c(block_table, np.int32)
    return int(lib().orc_slot(_ptr(bt), bt.size, int(block_size), int(num_blocks), int(p)))


def kv_encode(vals_bf16, scale):
    v = _c(vals_bf16, np.uint16)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_kv_encode(_ptr(v), v.size, float(scale), _ptr(out))
    return out


def prefill_rows(embed, tokens, hidden, w_norm_embed, w_norm_hidden, eps, fc, wk, wv,
                 nkv, hd, rope_base, rope_pos, cache_start, block_table, block_size,
                 num_blocks, k_scale, v_scale, rows, norm_mode=0, k_norm=None, in_norm=None):
    """Oracle K/V cache entries for the listed prompt rows (k_norm: per-head k norm
    weights [hd]; in_norm: the input norm weights [h] applied to y before k and v).

    Returns dict with y [n,h], k_rot [n,nkv*hd], v [n,nkv*hd] (bf16 bits), k_codes,
    v_codes [n,nkv*hd] (u8), slot [n] (int64, -1 = not written) and flags.
    """
    embed = _c(embed, np.uint16)
    hidden = _c(hidden, np.uint16)
    h = hidden.shape[1]
    rows = _c(rows, np.int64)
    n = rows.size
    kvd = nkv * hd
    y = np.empty((n, h), dtype=np.uint16)
    k_rot = np.empty((n, kvd), dtype=np.uint16)
    v = np.empty((n, kvd), dtype=np.uint16)
    kc = np.empty((n, kvd), dtype=np.uint8)
    vc = np.empty((n, kvd), dtype=np.uint8)
    sl = np.empty((n,), dtype=np.int64)
    bt = _c(block_table, np.int32)
    kn = None if k_norm is None else _c(k_norm, np.uint16)
    inn = None if in_norm is None else _c(in_norm, np.uint16)
    flags = lib().orc_prefill_rows_ext(
        _ptr(embed), embed.shape[0], _ptr(_c(tokens, np.int32)), _ptr(hidden), h,
        _ptr(_c(w_norm_embed, np.uint16)), _ptr(_c(w_norm_hidden, np.uint16)), float(eps),
        _ptr(_c(fc, np.uint16)), _ptr(_c(wk, np.uint16)), _ptr(_c(wv, np.uint16)), nkv, hd,
        float(rope_base), _ptr(_c(rope_pos, np.int32)), int(cache_start), _ptr(bt), bt.size,
        int(block_size), int(num_blocks), float(k_scale), float(v_scale), int(norm_mode),
        _ptr(kn), _ptr(inn), _ptr(rows), n, _ptr(y), _ptr(k_rot), _ptr(v), _ptr(kc), _ptr(vc), _ptr(sl))
    return dict(y=y, k_rot=k_rot, v=v, k_codes=kc, v_codes=vc, slot=sl, flags=int(flags))


# ---- decode attention (attn.c) ----------------------------------------------------

def paged_decode_attn(q, nkv, k_cache, v_cache, block_table, block_size, num_blocks, seq_len,
                      k_scale=1.0, v_scale=1.0, scale=None):
    """Single-token attention of q [nq, hd] (bf16 bits) over cache rows 0 .. seq_len - 1
    of an E4M3 cache [num_blocks, bs, nkv, hd]; scale defaults to 1/sqrt(hd). Returns
    (out [nq, hd] float64, flags)."""
    q = _c(q, np.uint16)
    nq, hd = q.shape
    scale = 1.0 / np.sqrt(hd) if scale is None else float(scale)
    kc = _c(k_cache, np.uint8)
    vc = _c(v_cache, np.uint8)
    bt = _c(block_table, np.int32)
    out = np.empty((nq, hd), dtype=np.float64)
    flags = lib().orc_paged_decode_attn(_ptr(q), nq, int(nkv), hd, _ptr(kc), _ptr(vc), _ptr(bt),
                                        bt.size, int(block_size), int(num_blocks), int(seq_len),
                                        float(k_scale), float(v_scale), scale, _ptr(out))
    return out, int(flags)


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
