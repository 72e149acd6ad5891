"""The C ABI without a GPU: the library loads, exports every symbol include/mtp.h
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes as C
import os
import re

import pytest

from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mtp_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(L.EXPORTS) == names


def test_version_and_status_strings(lib):
    assert L.mtp_abi_version() == 2
    for s in range(6):
        assert L.status_str(s)
    assert L.mtp_devflags_status(0) == L.MTP_OK
    assert L.mtp_devflags_status(L.MTP_DEVFLAG_EMPTY_MASK) == L.MTP_WARN_EMPTY_MASK
    assert L.mtp_devflags_status(L.MTP_DEVFLAG_BAD_TOKEN) == L.MTP_ERR_INVALID_ARG


# Fake 256-byte-aligned addresses: every call below fails validation first, so they
# are never dereferenced and no CUDA call is made.
A = 0x10000
B2 = 0x20000
OUT = 0x30000


def st(name, *args):
    return L.raw_status(name, *args)


def test_quantize_fp8_rejects(lib):
    assert st("mtp_quantize_fp8", None, 4, 32, OUT, OUT, None) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_quantize_fp8", A, 4, 24, OUT, OUT, None) == L.MTP_ERR_INVALID_ARG  # k % 16
    assert st("mtp_quantize_fp8", A, 0, 32, OUT, OUT, None) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_quantize_fp8", A + 2, 4, 32, OUT, OUT, None) == L.MTP_ERR_INVALID_ARG


def test_quantize_nvfp4_rejects(lib):
    ws_need = L.mtp_quantize_nvfp4_ws_bytes(4, 64)
    assert ws_need >= 256
    assert st("mtp_quantize_nvfp4", A, 4, 48, OUT, OUT, OUT, B2, ws_need, None) == \
        L.MTP_ERR_INVALID_ARG  # k % 32
    assert st("mtp_quantize_nvfp4", A, 4, 64, OUT, OUT, OUT, None, ws_need, None) == \
        L.MTP_ERR_WORKSPACE
    assert st("mtp_quantize_nvfp4", A, 4, 64, OUT, OUT, OUT, B2, ws_need - 1, None) == \
        L.MTP_ERR_WORKSPACE


def weight(fmt=L.MTP_FMT_BF16, n=100, k=64, data=A, rs=None, bs=None, gs=None):
    return L.mtp_weight(fmt, 0, n, k, data, rs, bs, gs)


def lm(head, n_eff=100, x=B2, M=1, mask=None, mw=0, ms=0, idx=OUT, ws=0x40000, wsb=None):
    if wsb is None:
        wsb = L.mtp_lm_head_ws_bytes(head, n_eff, M)
    return st("mtp_lm_head_argmax", C.byref(head), n_eff, x, M, mask, mw, ms, idx, None, None,
              None, ws, wsb, None)


def test_lm_head_rejects(lib):
    assert st("mtp_lm_head_argmax", None, 1, B2, 1, None, 0, 0, OUT, None, None, None,
              0x40000, 1 << 20, None) == L.MTP_ERR_INVALID_ARG
    assert lm(weight(k=60)) == L.MTP_ERR_INVALID_ARG             # bf16 k % 8
    assert lm(weight(fmt=1, k=40, rs=OUT)) == L.MTP_ERR_INVALID_ARG  # fp8 k % 16
    assert lm(weight(fmt=1, k=64)) == L.MTP_ERR_INVALID_ARG       # fp8 needs row scales
    assert lm(weight(fmt=2, k=48, bs=OUT, gs=OUT)) == L.MTP_ERR_INVALID_ARG  # nvfp4 k % 32
    assert lm(weight(fmt=2, k=64, bs=OUT)) == L.MTP_ERR_INVALID_ARG  # no global scale
    assert lm(weight(fmt=0, k=64, rs=OUT)) == L.MTP_ERR_INVALID_ARG  # stray pointer
    assert lm(weight(fmt=7)) == L.MTP_ERR_INVALID_ARG
    assert lm(weight(data=A + 8)) == L.MTP_ERR_INVALID_ARG        # 16-byte alignment
    assert lm(weight(), n_eff=101) == L.MTP_ERR_INVALID_ARG       # n_eff > n
    assert lm(weight(), n_eff=0) == L.MTP_ERR_INVALID_ARG
    assert lm(weight(), M=0) == L.MTP_ERR_UNSUPPORTED
    assert lm(weight(), M=33) == L.MTP_ERR_UNSUPPORTED
    assert lm(weight(), x=B2 + 4) == L.MTP_ERR_INVALID_ARG
    assert lm(weight(), mask=OUT, mw=0) == L.MTP_ERR_INVALID_ARG
    assert lm(weight(), ws=None) == L.MTP_ERR_WORKSPACE
    assert lm(weight(), wsb=16) == L.MTP_ERR_WORKSPACE
    # table rows must be a multiple of 128 bytes (the sweep streams 128-byte segments)
    assert lm(weight(k=40)) == L.MTP_ERR_UNSUPPORTED
    assert lm(weight(fmt=1, k=80, rs=OUT)) == L.MTP_ERR_UNSUPPORTED
    assert lm(weight(fmt=2, k=224, bs=OUT, gs=OUT)) == L.MTP_ERR_UNSUPPORTED
    # staged inputs larger than shared memory
    assert lm(weight(n=100, k=16384), M=8) == L.MTP_ERR_UNSUPPORTED
    # more than eight inputs stream x per K chunk, so the same width is fine there
    assert lm(weight(n=100, k=16384), M=16, ws=None) == L.MTP_ERR_WORKSPACE
    w = weight()
    w.reserved = 1
    assert lm(w) == L.MTP_ERR_INVALID_ARG


def test_lm_head_lp_rejects(lib):
    head = weight()
    wsb = L.mtp_lm_head_ws_bytes(head, 100, 1)

    def lp(out_lp, x=B2, n_eff=100):
        return st("mtp_lm_head_argmax_lp", C.byref(head), n_eff, x, 1, None, 0, 0, OUT, None,
                  out_lp, None, None, 0x40000, wsb, None)

    assert lp(None) == L.MTP_ERR_INVALID_ARG        # the log-probability output is required
    assert lp(OUT + 2) == L.MTP_ERR_INVALID_ARG     # f32 alignment
    assert lp(OUT, x=B2 + 4) == L.MTP_ERR_INVALID_ARG  # the same checks as mtp_lm_head_argmax
    assert lp(OUT, n_eff=101) == L.MTP_ERR_INVALID_ARG
    # partials are 16 bytes (max, index, sum of exponentials) for up to 1,024 CTAs x 32 inputs
    assert wsb == 256 + 16 * 32 * 1024
    # the no-alloc array adds 448 KB for x in the quantized sweeps' forms
    assert L.mtp_noalloc_scratch_bytes() == wsb + 448 * 1024
    up = lambda b: (b + 1023) // 1024 * 1024
    # quantized tables add x as their sweeps read it (+ 1 KB of exponents): FP8 from 7
    # inputs, two E4M3 planes of 16 or 32 rows; NVFP4 from 3 inputs, N = 6 MP rows of E2M1
    # terms (MP = 4, 8, 16, 32, rounded up to 16 rows) and their E4M3 block scales
    fp8 = weight(fmt=1, k=128, rs=OUT)
    assert L.mtp_lm_head_ws_bytes(fp8, 100, 6) == wsb  # FP8 streams x from 7 inputs on
    assert L.mtp_lm_head_ws_bytes(fp8, 100, 7) == wsb + 2 * 16 * 128 + 1024
    assert L.mtp_lm_head_ws_bytes(fp8, 100, 9) == wsb + 2 * 16 * 128 + 1024
    assert L.mtp_lm_head_ws_bytes(fp8, 100, 17) == wsb + 2 * 32 * 128 + 1024
    nv = weight(fmt=2, k=256, bs=OUT, gs=OUT)
    assert L.mtp_lm_head_ws_bytes(nv, 100, 1) == wsb and L.mtp_lm_head_ws_bytes(nv, 100, 2) == wsb
    for M, N in ((3, 32), (4, 32), (8, 48), (9, 96), (16, 96), (17, 192), (32, 192)):
        assert L.mtp_lm_head_ws_bytes(nv, 100, M) == wsb + up(N * 128) + up(N * 16) + 1024, M
    assert L.mtp_lm_head_ws_bytes(weight(k=128), 100, 32) == wsb
    # calls past the no-alloc array are rejected before any CUDA call
    noalloc = lambda head, M: st("mtp_lm_head_argmax_noalloc", C.byref(head), 100, B2, M, None,
                                 0, 0, OUT, None, None, None, None)
    assert noalloc(weight(fmt=1, k=14336, rs=OUT), 7) == L.MTP_ERR_WORKSPACE
    assert noalloc(weight(fmt=1, k=7168, rs=OUT), 17) == L.MTP_ERR_WORKSPACE
    assert noalloc(weight(fmt=2, k=8704, bs=OUT, gs=OUT), 16) == L.MTP_ERR_WORKSPACE
    assert noalloc(weight(fmt=2, k=4352, bs=OUT, gs=OUT), 32) == L.MTP_ERR_WORKSPACE
    # the table descriptor is checked before its size is looked at: a bad format, a bad k
    # or a missing scale is an argument error, not a workspace one
    assert noalloc(weight(fmt=7, k=128), 12) == L.MTP_ERR_INVALID_ARG
    assert noalloc(weight(fmt=1, k=100, rs=OUT), 7) == L.MTP_ERR_INVALID_ARG
    assert noalloc(weight(fmt=2, k=256, bs=OUT), 12) == L.MTP_ERR_INVALID_ARG
    # rows that are not a whole number of 128-byte segments are unsupported, at any M
    assert noalloc(weight(fmt=2, k=128, bs=OUT, gs=OUT), 12) == L.MTP_ERR_UNSUPPORTED


def test_lm_head_host_rejects(lib):
    head = weight()
    wsb = L.mtp_lm_head_host_ws_bytes(head, 100, 2)
    # the sweep's workspace, then the device copy of x (M k 2 bytes, 16-byte multiple)
    assert wsb == L.mtp_lm_head_ws_bytes(head, 100, 2) + 2 * 64 * 2

    def host(x=B2, out=OUT, M=2, ws=0x40000, nb=wsb):
        return st("mtp_lm_head_argmax_host", C.byref(head), 100, x, M, None, 0, 0, out, None,
                  ws, nb, None)

    assert host(x=None) == L.MTP_ERR_INVALID_ARG
    assert host(out=None) == L.MTP_ERR_INVALID_ARG
    assert host(M=33) == L.MTP_ERR_UNSUPPORTED
    assert host(x=B2 + 4) == L.MTP_ERR_INVALID_ARG
    assert host(out=OUT + 2) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_lm_head_argmax_host", None, 100, B2, 2, None, 0, 0, OUT, None, 0x40000, wsb,
              None) == L.MTP_ERR_INVALID_ARG  # no table
    assert host(ws=None) == L.MTP_ERR_WORKSPACE
    assert host(nb=wsb - 16) == L.MTP_ERR_WORKSPACE
    # addresses that are not pinned host memory (here: no device at all) are refused
    assert host() == L.MTP_ERR_INVALID_ARG


def test_shard_and_merge_rejects(lib):
    head = weight()
    wsb = L.mtp_lm_head_ws_bytes(head, 100, 1)

    def shard(part, off=0, n_eff=100):
        return st("mtp_lm_head_shard_partial", C.byref(head), n_eff, off, B2, 1, None, 0, 0,
                  part, None, None, 0x40000, wsb, None)

    assert shard(None) == L.MTP_ERR_INVALID_ARG          # the partial output is required
    assert shard(OUT + 8) == L.MTP_ERR_INVALID_ARG       # 16-byte aligned partials
    assert shard(OUT, off=-16) == L.MTP_ERR_INVALID_ARG
    assert shard(OUT, off=2**31 - 50) == L.MTP_ERR_INVALID_ARG  # global rows must fit i32
    assert shard(OUT, n_eff=101) == L.MTP_ERR_INVALID_ARG

    def merge(parts, n, M, idx=OUT):
        return st("mtp_argmax_merge_partials", parts, n, M, idx, None, None, None, None)

    assert merge(None, 2, 1) == L.MTP_ERR_INVALID_ARG
    assert merge(A, 0, 1) == L.MTP_ERR_INVALID_ARG
    assert merge(A, 2, 1, idx=None) == L.MTP_ERR_INVALID_ARG
    assert merge(A + 8, 2, 1) == L.MTP_ERR_INVALID_ARG
    assert merge(A, 2, 0) == L.MTP_ERR_UNSUPPORTED
    assert merge(A, 2, 33) == L.MTP_ERR_UNSUPPORTED


def test_combine_rejects(lib):
    fc = weight(n=32, k=64)
    args = [A, 50, B2, B2, 1, 32, OUT, OUT, 1e-6, 0, C.byref(fc), OUT, None, None]
    bad = list(args)
    bad[0] = None
    assert st("mtp_combine", *bad) == L.MTP_ERR_INVALID_ARG
    bad = list(args)
    bad[4] = 17
    assert st("mtp_combine", *bad) == L.MTP_ERR_UNSUPPORTED
    bad = list(args)
    bad[5] = 48
    fc48 = weight(n=48, k=96)  # 192-byte fc rows: not a multiple of 128
    bad[10] = C.byref(fc48)
    assert st("mtp_combine", *bad) == L.MTP_ERR_UNSUPPORTED
    bad = list(args)
    bad[5] = 24  # h % 16
    assert st("mtp_combine", *bad) == L.MTP_ERR_INVALID_ARG
    fc2 = weight(n=32, k=32)  # fc must be [h, 2h]
    bad = list(args)
    bad[10] = C.byref(fc2)
    assert st("mtp_combine", *bad) == L.MTP_ERR_INVALID_ARG
    bad = list(args)
    bad[8] = -1.0
    assert st("mtp_combine", *bad) == L.MTP_ERR_INVALID_ARG
    bad = list(args)
    bad[9] = 2  # norm_mode is MTP_NORM_W or MTP_NORM_ONE_PLUS_W
    assert st("mtp_combine", *bad) == L.MTP_ERR_INVALID_ARG


def test_debug_encoders_reject(lib):
    assert st("mtp_debug_encode_e4m3", None, 4, OUT, None) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_debug_encode_e2m1", A, 0, OUT, None) == L.MTP_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(OSError):
        L.load(str(tmp_path / "none.so"))


def prefill_args(**kw):
    a = dict(embed=A, vocab=100, tok=B2, hidden=A, R=10, h=256, wne=OUT, wnh=OUT, eps=1e-6,
             mode=0, fc=A, wk=A, wv=A, kn=None, inn=None, nkv=2, hd=128, base=1e6, pos=B2, start=0, table=B2, n_table=4,
             bs=16, kc=OUT, vc=OUT, nb=4, ks=1.0, vs=1.0, chunk=8, ws=0x100000, wsb=None,
             err=None)
    a.update(kw)
    if a["wsb"] is None:
        a["wsb"] = L.mtp_prefill_ws_bytes(min(a["chunk"], a["R"]), a["h"], a["nkv"], a["hd"])
    return [a[k] for k in ("embed", "vocab", "tok", "hidden", "R", "h", "wne", "wnh", "eps",
                           "mode", "fc", "wk", "wv", "kn", "inn", "nkv", "hd", "base", "pos", "start", "table",
                           "n_table", "bs", "kc", "vc", "nb", "ks", "vs", "chunk", "ws", "wsb",
                           "err")] + [None]


def test_prefill_rejects(lib):
    assert L.mtp_prefill_ws_bytes(2048, 5120, 8, 128) >= 2048 * 5120 * 6
    assert st("mtp_prefill_kv", *prefill_args(embed=None)) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_prefill_kv", *prefill_args(R=0)) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_prefill_kv", *prefill_args(ks=0.0)) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_prefill_kv", *prefill_args(mode=-1)) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_prefill_kv", *prefill_args(kn=OUT + 1)) == L.MTP_ERR_INVALID_ARG  # 2-byte
    assert st("mtp_prefill_kv", *prefill_args(inn=OUT + 8)) == L.MTP_ERR_INVALID_ARG  # 16-byte
    assert st("mtp_prefill_kv", *prefill_args(h=320)) == L.MTP_ERR_UNSUPPORTED   # h % 256
    assert st("mtp_prefill_kv", *prefill_args(hd=96)) == L.MTP_ERR_UNSUPPORTED
    # hidden sizes up to 12,288
    assert st("mtp_prefill_kv", *prefill_args(h=12544)) == L.MTP_ERR_UNSUPPORTED
    assert st("mtp_prefill_kv", *prefill_args(nkv=1)) == L.MTP_ERR_UNSUPPORTED  # nkv*hd % 256
    assert st("mtp_prefill_kv", *prefill_args(hidden=A + 8)) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_prefill_kv", *prefill_args(ws=None)) == L.MTP_ERR_WORKSPACE
    assert st("mtp_prefill_kv", *prefill_args(ws=0x100000 + 512)) == L.MTP_ERR_WORKSPACE
    assert st("mtp_prefill_kv", *prefill_args(wsb=1024)) == L.MTP_ERR_WORKSPACE
    # the recommended workspace is two chunk lanes; one lane is the minimum
    full = L.mtp_prefill_ws_bytes(8, 256, 2, 128)
    assert full % 2 == 0
    assert st("mtp_prefill_kv", *prefill_args(wsb=full // 2 - 1024)) == L.MTP_ERR_WORKSPACE


def test_gemm_and_kv_stage_reject(lib):
    assert st("mtp_debug_gemm_bf16", A, B2, OUT, 128, 100, 64, None) == L.MTP_ERR_UNSUPPORTED
    assert st("mtp_debug_gemm_bf16", A, B2, OUT, 128, 256, 48, None) == L.MTP_ERR_UNSUPPORTED
    assert st("mtp_debug_gemm_bf16", None, B2, OUT, 128, 256, 64, None) == L.MTP_ERR_INVALID_ARG
    assert st("mtp_debug_kv_write", A, B2, 10, 2, 100, 0, B2, 4, 16, 4, OUT, OUT, 1.0, 1.0,
              None, None) == L.MTP_ERR_INVALID_ARG  # hd % 32


def test_wait_timeout_rejects(lib):
    w = lambda which, lim, ctr=OUT, err=OUT: st("mtp_debug_wait_timeout", which, lim, ctr, err, None)
    assert w(2, 1000) == L.MTP_ERR_INVALID_ARG          # which is 0 or 1
    assert w(0, 0) == L.MTP_ERR_INVALID_ARG             # limit in [1, 4e9] cycles
    assert w(0, 5_000_000_000) == L.MTP_ERR_INVALID_ARG
    assert w(0, 1000, err=None) == L.MTP_ERR_INVALID_ARG  # the error word is required
    assert w(1, 1000, ctr=None) == L.MTP_ERR_INVALID_ARG  # the counter wait needs its counter
    assert w(1, 1000, ctr=OUT + 2) == L.MTP_ERR_INVALID_ARG


def test_draft_step_rejects(lib):
    def ds(M=1, h=256, embed=A, head=B2, mask=None, mw=0, ms=0, idx=OUT, n=100, mode=0, y=None,
           hid=A):
        return st("mtp_draft_step", embed, 100, OUT, hid, M, h, A, A, 1e-6, mode, A, head, n, mask,
                  mw, ms, y, idx, None, None, None)
    assert ds(embed=None) == L.MTP_ERR_INVALID_ARG
    assert ds(idx=None) == L.MTP_ERR_INVALID_ARG
    assert ds(h=260) == L.MTP_ERR_INVALID_ARG       # h % 8
    assert ds(n=0) == L.MTP_ERR_INVALID_ARG
    assert ds(mode=3) == L.MTP_ERR_INVALID_ARG
    assert ds(mask=OUT, mw=0) == L.MTP_ERR_INVALID_ARG
    assert ds(M=5) == L.MTP_ERR_UNSUPPORTED         # up to 4 inputs
    assert ds(h=2048) == L.MTP_ERR_UNSUPPORTED      # up to hidden 1024
    assert ds(head=B2 + 8) == L.MTP_ERR_INVALID_ARG  # 16-byte aligned head
    assert ds(y=A) == L.MTP_ERR_INVALID_ARG          # out_y must not overlap hidden
    assert ds(y=A + 510, h=256) == L.MTP_ERR_INVALID_ARG
    assert ds(y=A - 510, h=256) == L.MTP_ERR_INVALID_ARG


def test_paged_decode_attn_rejects(lib):
    ws = L.mtp_paged_decode_attn_ws_bytes(8, 128, 300)
    # up to one piece per 64 cache rows: 5 pieces x heads x (hd + max + sum) floats
    assert ws == 5 * 8 * 130 * 4
    assert L.mtp_paged_decode_attn_ws_bytes(8, 128, 2_000_000) == 1024 * 8 * 130 * 4  # at most 1,024

    def at(q=A, nq=8, nkv=2, hd=128, seq=300, ks=1.0, sc=0.1, w=0x40000, wb=ws, kc=B2):
        return st("mtp_paged_decode_attn", q, nq, nkv, hd, kc, B2, OUT, 20, 16, 30, seq, ks, 1.0,
                  sc, OUT, None, w, wb, None)
    assert at(q=None) == L.MTP_ERR_INVALID_ARG
    assert at(nq=9) == L.MTP_ERR_INVALID_ARG        # nq % nkv
    assert at(seq=0) == L.MTP_ERR_INVALID_ARG
    assert at(ks=0.0) == L.MTP_ERR_INVALID_ARG
    assert at(sc=-1.0) == L.MTP_ERR_INVALID_ARG
    assert at(hd=96) == L.MTP_ERR_UNSUPPORTED
    assert at(nq=34, nkv=2) == L.MTP_ERR_UNSUPPORTED  # at most 16 query heads per kv head
    assert at(kc=B2 + 8) == L.MTP_ERR_INVALID_ARG
    assert at(w=None) == L.MTP_ERR_WORKSPACE
    assert at(wb=ws - 4) == L.MTP_ERR_WORKSPACE
