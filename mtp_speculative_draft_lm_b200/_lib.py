"""ctypes binding of ``libmtp.so`` (include/mtp.h): argument marshalling only.

Every function here has the C entry point's name and arguments. Pointer arguments
accept a torch tensor (its ``data_ptr()``), a plain integer address, or None for
NULL; ``stream`` defaults to torch's current CUDA stream. A non-zero status raises
:class:`MtpError`. There is no fallback: if the library is missing, loading it
raises.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmtp.so")

MTP_OK = 0
MTP_ERR_INVALID_ARG = 1
MTP_ERR_UNSUPPORTED = 2
MTP_ERR_WORKSPACE = 3
MTP_ERR_CUDA = 4
MTP_WARN_EMPTY_MASK = 5

MTP_DEVFLAG_BAD_TOKEN = 1
MTP_DEVFLAG_EMPTY_MASK = 2
MTP_DEVFLAG_BAD_SLOT = 4
MTP_DEVFLAG_TIMEOUT = 8

MTP_NORM_W = 0
MTP_NORM_ONE_PLUS_W = 1

MTP_FMT_BF16 = 0
MTP_FMT_FP8_ROW = 1
MTP_FMT_NVFP4 = 2

#: every symbol include/mtp.h declares
EXPORTS = (
    "mtp_abi_version", "mtp_status_str", "mtp_devflags_status",
    "mtp_quantize_fp8", "mtp_quantize_nvfp4_ws_bytes", "mtp_quantize_nvfp4",
    "mtp_combine", "mtp_lm_head_ws_bytes", "mtp_lm_head_argmax", "mtp_lm_head_argmax_lp",
    "mtp_lm_head_host_ws_bytes", "mtp_lm_head_argmax_host",
    "mtp_lm_head_shard_partial", "mtp_argmax_merge_partials",
    "mtp_debug_encode_e4m3", "mtp_debug_encode_e2m1", "mtp_nvfp4_scale_pitch",
    "mtp_debug_wait_timeout", "mtp_draft_step", "mtp_paged_decode_attn_ws_bytes",
    "mtp_paged_decode_attn",
    "mtp_noalloc_scratch_bytes", "mtp_lm_head_argmax_noalloc",
    "mtp_prefill_ws_bytes", "mtp_prefill_kv", "mtp_debug_gemm_bf16", "mtp_debug_kv_write",
)


class MtpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_str(status)})")


class mtp_weight(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("reserved", C.c_int32), ("n", C.c_int64),
                ("k", C.c_int64), ("data", C.c_void_p), ("row_scale", C.c_void_p),
                ("block_scale", C.c_void_p), ("global_scale", C.c_void_p)]


_P = C.c_void_p
_I32 = C.c_int32
_I64 = C.c_int64
_SZ = C.c_size_t
_W = C.POINTER(mtp_weight)

_SIGS = {
    "mtp_abi_version": (_I32, []),
    "mtp_status_str": (C.c_char_p, [C.c_int]),
    "mtp_devflags_status": (C.c_int, [_I32]),
    "mtp_quantize_fp8": (C.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "mtp_quantize_nvfp4_ws_bytes": (_SZ, [_I64, _I64]),
    "mtp_nvfp4_scale_pitch": (_I64, [_I64]),
    "mtp_quantize_nvfp4": (C.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "mtp_combine": (C.c_int, [_P, _I64, _P, _P, _I32, _I32, _P, _P, C.c_float, _I32, _W, _P,
                              _P, _P]),
    "mtp_lm_head_ws_bytes": (_SZ, [_W, _I64, _I32]),
    "mtp_lm_head_argmax": (C.c_int, [_W, _I64, _P, _I32, _P, _I64, _I64, _P, _P, _P, _P,
                                     _P, _SZ, _P]),
    "mtp_lm_head_argmax_lp": (C.c_int, [_W, _I64, _P, _I32, _P, _I64, _I64, _P, _P, _P, _P,
                                        _P, _P, _SZ, _P]),
    "mtp_lm_head_host_ws_bytes": (_SZ, [_W, _I64, _I32]),
    "mtp_lm_head_argmax_host": (C.c_int, [_W, _I64, _P, _I32, _P, _I64, _I64, _P, _P, _P, _SZ,
                                          _P]),
    "mtp_lm_head_shard_partial": (C.c_int, [_W, _I64, _I64, _P, _I32, _P, _I64, _I64, _P, _P,
                                            _P, _P, _SZ, _P]),
    "mtp_argmax_merge_partials": (C.c_int, [_P, _I32, _I32, _P, _P, _P, _P, _P]),
    "mtp_prefill_ws_bytes": (_SZ, [_I64, _I32, _I32, _I32]),
    "mtp_prefill_kv": (C.c_int, [_P, _I64, _P, _P, _I64, _I32, _P, _P, C.c_float, _I32, _P, _P,
                                 _P, _P, _P, _I32, _I32, C.c_float, _P, _I64, _P, _I64, _I32, _P, _P,
                                 _I64, C.c_float, C.c_float, _I64, _P, _SZ, _P, _P]),
    "mtp_debug_gemm_bf16": (C.c_int, [_P, _P, _P, _I32, _I32, _I32, _P]),
    "mtp_debug_kv_write": (C.c_int, [_P, _P, _I64, _I32, _I32, _I64, _P, _I64, _I32, _I64, _P,
                                     _P, C.c_float, C.c_float, _P, _P]),
    "mtp_noalloc_scratch_bytes": (_SZ, []),
    "mtp_lm_head_argmax_noalloc": (C.c_int, [_W, _I64, _P, _I32, _P, _I64, _I64, _P, _P, _P,
                                             _P, _P]),
    "mtp_debug_wait_timeout": (C.c_int, [_I32, _I64, _P, _P, _P]),
    "mtp_paged_decode_attn_ws_bytes": (_SZ, [_I32, _I32, _I64]),
    "mtp_paged_decode_attn": (C.c_int, [_P, _I32, _I32, _I32, _P, _P, _P, _I64, _I32, _I64,
                                        _I64, C.c_float, C.c_float, C.c_float, _P, _P, _P, _SZ,
                                        _P]),
    "mtp_draft_step": (C.c_int, [_P, _I64, _P, _P, _I32, _I32, _P, _P, C.c_float, _I32, _P, _P,
                                 _I64, _P, _I64, _I64, _P, _P, _P, _P, _P]),
    "mtp_debug_encode_e4m3": (C.c_int, [_P, _I64, _P, _P]),
    "mtp_debug_encode_e2m1": (C.c_int, [_P, _I64, _P, _P]),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libmtp.so (raises OSError if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} not found: build it with mtp_speculative_draft_lm_b200.build")
        lib = C.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s):
    if s is None:
        import torch

        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str):
    if st != MTP_OK:
        raise MtpError(st, where)


def status_str(st: int) -> str:
    return load().mtp_status_str(st).decode()


def weight(fmt: int, n: int, k: int, data, row_scale=None, block_scale=None,
           global_scale=None) -> mtp_weight:
    return mtp_weight(int(fmt), 0, int(n), int(k), _ptr(data), _ptr(row_scale),
                      _ptr(block_scale), _ptr(global_scale))


def mtp_abi_version() -> int:
    return load().mtp_abi_version()


def mtp_devflags_status(value: int) -> int:
    return load().mtp_devflags_status(int(value))


def mtp_quantize_fp8(w, n, k, codes, row_scale, stream=None):
    _check(load().mtp_quantize_fp8(_ptr(w), n, k, _ptr(codes), _ptr(row_scale),
                                   _stream(stream)), "mtp_quantize_fp8")


def mtp_nvfp4_scale_pitch(k) -> int:
    return load().mtp_nvfp4_scale_pitch(k)


def mtp_quantize_nvfp4_ws_bytes(n, k) -> int:
    return load().mtp_quantize_nvfp4_ws_bytes(n, k)


def mtp_quantize_nvfp4(w, n, k, codes, block_scale, global_scale, ws, ws_bytes, stream=None):
    _check(load().mtp_quantize_nvfp4(_ptr(w), n, k, _ptr(codes), _ptr(block_scale),
                                     _ptr(global_scale), _ptr(ws), ws_bytes, _stream(stream)),
           "mtp_quantize_nvfp4")


def mtp_combine(embed, vocab, token_ids, hidden, M, h, w_norm_embed, w_norm_hidden, eps,
                norm_mode, fc, out, dev_err=None, stream=None):
    _check(load().mtp_combine(_ptr(embed), vocab, _ptr(token_ids), _ptr(hidden), M, h,
                              _ptr(w_norm_embed), _ptr(w_norm_hidden), float(eps), int(norm_mode),
                              C.byref(fc) if fc is not None else None, _ptr(out),
                              _ptr(dev_err), _stream(stream)), "mtp_combine")


def mtp_lm_head_ws_bytes(head, n_eff, M) -> int:
    return load().mtp_lm_head_ws_bytes(C.byref(head), n_eff, M)


def mtp_lm_head_argmax(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx,
                       out_val, out_logits, dev_err, ws, ws_bytes, stream=None):
    _check(load().mtp_lm_head_argmax(C.byref(head) if head is not None else None, n_eff,
                                     _ptr(x), M, _ptr(mask), mask_words, mask_stride_words,
                                     _ptr(out_idx), _ptr(out_val), _ptr(out_logits),
                                     _ptr(dev_err), _ptr(ws), ws_bytes, _stream(stream)),
           "mtp_lm_head_argmax")


def mtp_lm_head_argmax_lp(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx,
                          out_val, out_logprob, out_logits, dev_err, ws, ws_bytes, stream=None):
    _check(load().mtp_lm_head_argmax_lp(C.byref(head) if head is not None else None, n_eff,
                                        _ptr(x), M, _ptr(mask), mask_words, mask_stride_words,
                                        _ptr(out_idx), _ptr(out_val), _ptr(out_logprob),
                                        _ptr(out_logits), _ptr(dev_err), _ptr(ws), ws_bytes,
                                        _stream(stream)),
           "mtp_lm_head_argmax_lp")


def mtp_lm_head_host_ws_bytes(head, n_eff, M) -> int:
    return load().mtp_lm_head_host_ws_bytes(C.byref(head), n_eff, M)


def mtp_lm_head_argmax_host(head, n_eff, x_host, M, mask, mask_words, mask_stride_words,
                            out_host, dev_err, ws, ws_bytes, stream=None):
    _check(load().mtp_lm_head_argmax_host(C.byref(head) if head is not None else None, n_eff,
                                          _ptr(x_host), M, _ptr(mask), mask_words,
                                          mask_stride_words, _ptr(out_host), _ptr(dev_err),
                                          _ptr(ws), ws_bytes, _stream(stream)),
           "mtp_lm_head_argmax_host")


def mtp_lm_head_shard_partial(shard, n_eff, row_offset, x, M, mask, mask_words,
                              mask_stride_words, out_partial, out_logits, dev_err, ws, ws_bytes,
                              stream=None):
    _check(load().mtp_lm_head_shard_partial(C.byref(shard) if shard is not None else None,
                                            n_eff, row_offset, _ptr(x), M, _ptr(mask),
                                            mask_words, mask_stride_words, _ptr(out_partial),
                                            _ptr(out_logits), _ptr(dev_err), _ptr(ws), ws_bytes,
                                            _stream(stream)),
           "mtp_lm_head_shard_partial")


def mtp_argmax_merge_partials(partials, n_parts, M, out_idx, out_val, out_logprob, dev_err,
                              stream=None):
    _check(load().mtp_argmax_merge_partials(_ptr(partials), n_parts, M, _ptr(out_idx),
                                            _ptr(out_val), _ptr(out_logprob), _ptr(dev_err),
                                            _stream(stream)),
           "mtp_argmax_merge_partials")


def mtp_prefill_ws_bytes(chunk_rows, h, nkv, hd) -> int:
    return load().mtp_prefill_ws_bytes(chunk_rows, h, nkv, hd)


def mtp_prefill_kv(embed, vocab, token_ids, hidden, R, h, w_norm_embed, w_norm_hidden, eps,
                   norm_mode, fc, wk, wv, k_norm, in_norm, nkv, hd, rope_base, rope_pos,
                   cache_start,
                   block_table, n_table, block_size, k_cache, v_cache, num_blocks, k_scale,
                   v_scale, chunk_rows, ws, ws_bytes, dev_err=None, stream=None):
    _check(load().mtp_prefill_kv(_ptr(embed), vocab, _ptr(token_ids), _ptr(hidden), R, h,
                                 _ptr(w_norm_embed), _ptr(w_norm_hidden), float(eps),
                                 int(norm_mode), _ptr(fc), _ptr(wk), _ptr(wv), _ptr(k_norm),
                                 _ptr(in_norm), nkv,
                                 hd, float(rope_base), _ptr(rope_pos),
                                 cache_start, _ptr(block_table), n_table, block_size,
                                 _ptr(k_cache), _ptr(v_cache), num_blocks, float(k_scale),
                                 float(v_scale), chunk_rows, _ptr(ws), ws_bytes, _ptr(dev_err),
                                 _stream(stream)), "mtp_prefill_kv")


def mtp_debug_gemm_bf16(A, B, Cout, M, N, K, stream=None):
    _check(load().mtp_debug_gemm_bf16(_ptr(A), _ptr(B), _ptr(Cout), M, N, K, _stream(stream)),
           "mtp_debug_gemm_bf16")


def mtp_debug_kv_write(k_rot, v, R, nkv, hd, cache_start, block_table, n_table, block_size,
                       num_blocks, k_cache, v_cache, k_scale, v_scale, dev_err=None, stream=None):
    _check(load().mtp_debug_kv_write(_ptr(k_rot), _ptr(v), R, nkv, hd, cache_start,
                                     _ptr(block_table), n_table, block_size, num_blocks,
                                     _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale),
                                     _ptr(dev_err), _stream(stream)), "mtp_debug_kv_write")


def mtp_noalloc_scratch_bytes() -> int:
    return load().mtp_noalloc_scratch_bytes()


def mtp_lm_head_argmax_noalloc(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx,
                               out_val, out_logits, dev_err, stream=None):
    _check(load().mtp_lm_head_argmax_noalloc(C.byref(head) if head is not None else None, n_eff,
                                             _ptr(x), M, _ptr(mask), mask_words,
                                             mask_stride_words, _ptr(out_idx), _ptr(out_val),
                                             _ptr(out_logits), _ptr(dev_err), _stream(stream)),
           "mtp_lm_head_argmax_noalloc")


def mtp_draft_step(embed, vocab, token_ids, hidden, M, h, w_norm_embed, w_norm_hidden, eps,
                   norm_mode, fc, head, n_eff, mask, mask_words, mask_stride_words, out_y,
                   out_idx, out_val, dev_err=None, stream=None):
    _check(load().mtp_draft_step(_ptr(embed), vocab, _ptr(token_ids), _ptr(hidden), M, h,
                                 _ptr(w_norm_embed), _ptr(w_norm_hidden), float(eps),
                                 int(norm_mode), _ptr(fc),
                                 _ptr(head), n_eff, _ptr(mask), mask_words, mask_stride_words,
                                 _ptr(out_y), _ptr(out_idx), _ptr(out_val), _ptr(dev_err),
                                 _stream(stream)), "mtp_draft_step")


def mtp_paged_decode_attn_ws_bytes(nq, hd, seq_len) -> int:
    return load().mtp_paged_decode_attn_ws_bytes(nq, hd, seq_len)


def mtp_paged_decode_attn(q, nq, nkv, hd, k_cache, v_cache, block_table, n_table, block_size,
                          num_blocks, seq_len, k_scale, v_scale, scale, out, dev_err, ws, ws_bytes,
                          stream=None):
    _check(load().mtp_paged_decode_attn(_ptr(q), nq, nkv, hd, _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_table), n_table, block_size, num_blocks,
                                        seq_len, float(k_scale), float(v_scale), float(scale),
                                        _ptr(out), _ptr(dev_err), _ptr(ws), ws_bytes,
                                        _stream(stream)), "mtp_paged_decode_attn")


def mtp_debug_wait_timeout(which, limit_cycles, counter, dev_err, stream=None):
    _check(load().mtp_debug_wait_timeout(int(which), int(limit_cycles), _ptr(counter),
                                         _ptr(dev_err), _stream(stream)),
           "mtp_debug_wait_timeout")


def mtp_debug_encode_e4m3(inp, n, out, stream=None):
    _check(load().mtp_debug_encode_e4m3(_ptr(inp), n, _ptr(out), _stream(stream)),
           "mtp_debug_encode_e4m3")


def mtp_debug_encode_e2m1(inp, n, out, stream=None):
    _check(load().mtp_debug_encode_e2m1(_ptr(inp), n, _ptr(out), _stream(stream)),
           "mtp_debug_encode_e2m1")


def raw_status(name: str, *args) -> int:
    """Call an entry point and return its status without raising (for error tests)."""
    return getattr(load(), name)(*args)
