"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: brute force over
every code of a format, closed forms, invariants, hand-worked fixtures under
tests/golden/, or an independent library routine (torch's float8 cast, numpy's
float64 matmul). A plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong tie rule) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from mtp_speculative_draft_lm_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers (test-side)

def e4m3_table():
    """All 256 E4M3FN code values decoded by torch (independent of the oracle)."""
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    return t.astype(np.float64)


E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def brute_encode(v, mags, sat_code, sign_bit):
    """Nearest magnitude by linear search over every code, ties to the even code."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equal distances prefer the even code (lowest set bit clear)
    even = cand & (np.arange(mags.size)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    pick = np.where(a >= mags[sat_code], sat_code, pick)
    sign = np.signbit(v).astype(np.int64) * sign_bit
    return (pick | sign).astype(np.uint8)


def all_bf16_values():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32).astype(np.float64)
    return f[~np.isnan(f)]


def midpoints_with_neighbours(mags):
    mids = (mags[1:] + mags[:-1]) / 2
    f32 = mids.astype(np.float32)
    up = np.nextafter(f32, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(f32, np.float32(-np.inf)).astype(np.float64)
    v = np.concatenate([mids, up, dn])
    return np.concatenate([v, -v])


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def u16(t):
    return synth.as_u16(t)


# ---------------------------------------------------------------- formats

def test_e4m3_decode_matches_torch(orc):
    ref = e4m3_table()
    got = orc.e4m3_value(np.arange(256))
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], ref[finite])
    assert orc.e4m3_value([0x7E])[0] == 448.0
    assert orc.e4m3_value([0x01])[0] == 2.0 ** -9


def test_e4m3_encode_bruteforce_all_bf16_and_midpoints(orc):
    mags = e4m3_table()[:127]  # codes 0x00..0x7E, increasing
    assert np.all(np.diff(mags) > 0)
    v = np.concatenate([all_bf16_values(), midpoints_with_neighbours(mags),
                        [np.inf, -np.inf, 1e30, -1e30]])
    got = orc.e4m3_encode(v)
    ref = brute_encode(v, mags, 0x7E, 0x80)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_encode_matches_torch_cast(orc):
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-14, 9, (200000,),
                                                                    generator=g).float())
    x = x[x.abs() < 464]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_encode(x.double().numpy())
    assert np.array_equal(got, ref)


def test_e4m3_sign_and_saturation(orc):
    assert orc.e4m3_encode([-1e-12])[0] == 0x80
    assert orc.e4m3_encode([-0.0])[0] == 0x80
    assert orc.e4m3_encode([0.0])[0] == 0x00
    assert orc.e4m3_encode([448.0])[0] == 0x7E
    assert orc.e4m3_encode([1e9])[0] == 0x7E
    assert orc.e4m3_encode([-1e9])[0] == 0xFE
    # never the NaN pattern for finite input
    v = np.linspace(-1000, 1000, 100001)
    assert not np.any((orc.e4m3_encode(v) & 0x7F) == 0x7F)


def test_e2m1_encode_bruteforce_dense_grid(orc):
    grid = np.arange(-8 * 4096, 8 * 4096 + 1) / 4096.0
    v = np.concatenate([grid, midpoints_with_neighbours(E2M1_MAG)])
    got = orc.e2m1_encode(v)
    ref = brute_encode(v, E2M1_MAG, 7, 8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e2m1_tie_table(orc):
    # worked special cases: each midpoint goes to the even code
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        code = orc.e2m1_encode([v])[0]
        assert orc.e2m1_value([code])[0] == want, v
        assert orc.e2m1_value([orc.e2m1_encode([-v])[0]])[0] == -want
    assert orc.e2m1_encode([-0.1])[0] == 0x8
    assert orc.e2m1_encode([100.0])[0] == 0x7
    assert list(orc.e2m1_value(np.arange(8))) == list(E2M1_MAG)


def test_bf16_rounding(orc):
    g = torch.Generator().manual_seed(3)
    x = torch.randn(100000, generator=g) * 100
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f64_to_bf16(x.double().numpy()), ref)
    # single rounding from the real value: just above a bf16 midpoint rounds up,
    # although an fp32 intermediate would have made it an exact tie (-> even, down)
    assert orc.f64_to_bf16([1 + 2 ** -8 + 2 ** -30])[0] == 0x3F81
    assert orc.f64_to_bf16([1 + 2 ** -8])[0] == 0x3F80  # exact tie -> even
    assert orc.f64_to_bf16([-0.0])[0] == 0x8000


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector_is_the_weight(orc):
    h = 96
    w = u16(synth.normal_bf16(synth._gen(1), (h,), 0.1, 1.0))
    for c in (0.5, 3.0, -2.0):
        x = u16(bf16(np.full(h, c)))
        y = orc.rmsnorm(x, w, 0.0)
        want = w if c > 0 else (w ^ 0x8000)
        assert np.array_equal(y, want)


def test_rmsnorm_one_hot_and_scale_invariance(orc):
    h = 64  # sqrt(h) = 8, a power of two: exact
    w = u16(synth.normal_bf16(synth._gen(2), (h,), 0.1, 1.0))
    x = np.zeros(h, np.float32)
    x[17] = 0.37
    y = orc.rmsnorm(u16(bf16(x)), w, 0.0)
    wf = orc.bf16_to_f64(w)
    assert orc.bf16_to_f64(y)[17] == wf[17] * 8.0
    assert np.all(orc.bf16_to_f64(y)[np.arange(h) != 17] == 0)
    xr = u16(synth.normal_bf16(synth._gen(3), (h,), 1.0))
    x4 = orc.f64_to_bf16(orc.bf16_to_f64(xr) * 4.0)
    assert np.array_equal(orc.rmsnorm(xr, w, 0.0), orc.rmsnorm(x4, w, 0.0))


def test_rmsnorm_unit_rms_and_library(orc):
    h = 512
    ones = u16(bf16(np.ones(h)))
    x = u16(synth.normal_bf16(synth._gen(4), (h,), 3.0))
    y = orc.bf16_to_f64(orc.rmsnorm(x, ones, 0.0))
    assert abs(np.mean(y * y) - 1.0) < 2 ** -7
    xf = orc.bf16_to_f64(x)
    eps = 1e-6
    ref = xf / (np.linalg.norm(xf) / math.sqrt(h) * math.sqrt(1 + eps * h / np.dot(xf, xf)))
    assert np.allclose(y, ref, rtol=2 ** -8, atol=0)
    assert np.all(orc.rmsnorm(np.zeros(h, np.uint16), ones, 1e-6) == 0)


# ---------------------------------------------------------------- combiner

def tiny(h=32, vocab=50, M=3, seed=11):
    d = synth.tiny_draft(seed=seed, vocab=vocab, h=h, M=M)
    return {k: (u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else v)
            for k, v in d.items()}


def test_combine_one_hot_selects_fc_column(orc):
    d = tiny()
    h = d["h"]
    j = 5
    w_ne = np.zeros(h, np.float32)
    w_ne[j] = 1.0
    embed = d["embed"].copy()
    embed[3] = u16(bf16(np.full(h, 0.25)))
    y, concat, flags = orc.combine(embed, [3], d["hidden"][:1], u16(bf16(w_ne)),
                                   np.zeros(h, np.uint16), 0.0, d["fc"])
    assert flags == 0
    assert np.array_equal(y[0], d["fc"][:, j])
    assert np.all(orc.bf16_to_f64(concat[0, h:]) == 0)


def test_combine_embedding_half_only_and_order(orc):
    d = tiny()
    h = d["h"]
    y, concat, _ = orc.combine(d["embed"], d["tokens"], d["hidden"], d["w_norm_embed"],
                               np.zeros(h, np.uint16), d["eps"], d["fc"])
    for m in range(d["hidden"].shape[0]):
        ne = orc.rmsnorm(d["embed"][d["tokens"][m]], d["w_norm_embed"], d["eps"])
        assert np.array_equal(concat[m, :h], ne)
        ref = orc.bf16_to_f64(d["fc"])[:, :h] @ orc.bf16_to_f64(ne)
        assert np.array_equal(y[m], orc.f64_to_bf16(ref))


def test_combine_full_matches_numpy(orc):
    d = tiny(h=4, vocab=9, M=2)
    y, concat, _ = orc.combine(d["embed"], d["tokens"], d["hidden"], d["w_norm_embed"],
                               d["w_norm_hidden"], d["eps"], d["fc"])
    for m in range(2):
        nh = orc.rmsnorm(d["hidden"][m], d["w_norm_hidden"], d["eps"])
        assert np.array_equal(concat[m, 4:], nh)
        ref = orc.bf16_to_f64(d["fc"]) @ orc.bf16_to_f64(concat[m])
        assert np.array_equal(y[m], orc.f64_to_bf16(ref))


def test_combine_bad_token_flags_and_zeroes(orc):
    d = tiny()
    y, concat, flags = orc.combine(d["embed"], [d["vocab"]], d["hidden"][:1],
                                   d["w_norm_embed"], d["w_norm_hidden"], d["eps"], d["fc"])
    assert flags & orc.FLAG_BAD_TOKEN
    assert np.all(orc.bf16_to_f64(concat[0, : d["h"]]) == 0)


# ---------------------------------------------------------------- lm_head + argmax

def quantized(orc, W, fmt):
    if fmt == orc.FMT_BF16:
        return dict(data=W)
    if fmt == orc.FMT_FP8_ROW:
        c, s = orc.quantize_fp8(W)
        return dict(data=c, row_scale=s)
    c, b, g = orc.quantize_nvfp4(W)
    return dict(data=c, block_scale=b, global_scale=g)


def independent_dequant(orc, fmt, q, k):
    """Dequantize with torch's float8 decode and a literal E2M1 table."""
    if fmt == orc.FMT_BF16:
        return orc.bf16_to_f64(q["data"])
    t8 = e4m3_table()
    if fmt == orc.FMT_FP8_ROW:
        return t8[q["data"]] * q["row_scale"].astype(np.float64)[:, None]
    lo = q["data"] & 0xF
    hi = q["data"] >> 4
    codes = np.stack([lo, hi], axis=2).reshape(q["data"].shape[0], k)
    mag = E2M1_MAG[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sc = np.repeat(t8[q["block_scale"]], 16, axis=1)
    return mag * sc * np.float64(np.float32(q["global_scale"]))


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_lm_head_one_hot_selects_entries(orc, fmt):
    N, K = 37, 64
    W = u16(synth.normal_bf16(synth._gen(21), (N, K), 0.02))
    q = quantized(orc, W, fmt)
    deq = independent_dequant(orc, fmt, q, K)
    for j in (0, 17, K - 1):
        x = np.zeros(K, np.float32)
        x[j] = 1.0
        logits, _, _, _ = orc.lm_head_argmax(fmt, q["data"], K, u16(bf16(x)),
                                             row_scale=q.get("row_scale"),
                                             block_scale=q.get("block_scale"),
                                             global_scale=q.get("global_scale", 0.0))
        assert np.array_equal(logits[0], deq[:, j])


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_lm_head_matches_numpy_matmul(orc, fmt):
    N, K, M = 37, 32, 3
    W = u16(synth.normal_bf16(synth._gen(22), (N, K), 0.02))
    x = u16(synth.normal_bf16(synth._gen(23), (M, K), 1.0))
    q = quantized(orc, W, fmt)
    logits, idx, val, flags = orc.lm_head_argmax(fmt, q["data"], K, x,
                                                 row_scale=q.get("row_scale"),
                                                 block_scale=q.get("block_scale"),
                                                 global_scale=q.get("global_scale", 0.0))
    ref = orc.bf16_to_f64(x) @ independent_dequant(orc, fmt, q, K).T
    assert np.allclose(logits, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(idx, ref.argmax(axis=1)) and flags == 0
    assert np.array_equal(val, ref.max(axis=1))


def test_lm_head_n_eff_limits_rows(orc):
    d = synth.head_table(31, 200, 64, 2)
    W, x = u16(d["W"]), u16(d["x"])
    full, _, _, _ = orc.lm_head_argmax(0, W, 64, x)
    part, idx, _, _ = orc.lm_head_argmax(0, W, 64, x, n_eff=150)
    assert part.shape == (2, 150)
    assert np.array_equal(part, full[:, :150])
    assert np.array_equal(idx, full[:, :150].argmax(axis=1))


def test_argmax_planted_and_masked_decoy(orc):
    d = synth.head_table(41, 3000, 128, 4, mask_keep=0.1)
    W, x = u16(d["W"]), u16(d["x"])
    logits, idx, val, flags = orc.lm_head_argmax(0, W, 128, x)
    assert np.array_equal(idx, d["top"]) and flags == 0
    words = d["mask"].shape[1]
    mlog, midx, mval, mflags = orc.lm_head_argmax(0, W, 128, x, mask=d["mask"],
                                                  mask_words=words, mask_stride_words=words)
    assert np.array_equal(midx, d["second"]) and mflags == 0
    for m in range(4):
        assert mlog[m, d["top"][m]] > mval[m]  # the decoy is larger but masked
        allowed = d["allowed"][m]
        assert mval[m] == logits[m][allowed].max()
        srt = np.sort(logits[m])
        assert srt[-1] - srt[-2] >= 0.5  # planted gap


def test_argmax_ties_lowest_index_and_empty_mask(orc):
    d = synth.head_table(51, 100, 64, 1)
    W = u16(d["W"]).copy()
    top = int(d["top"][0])
    dup = [3, top, 60] if top > 3 else [top, 70, 80]
    for r in dup:
        W[r] = W[top]
    _, idx, _, _ = orc.lm_head_argmax(0, W, 64, u16(d["x"]))
    assert idx[0] == min(dup)
    # all tokens masked -> index 0, value -inf, flag
    mask = np.zeros((1, 4), np.int32)
    _, idx, val, flags = orc.lm_head_argmax(0, W, 64, u16(d["x"]), mask=mask, mask_words=4)
    assert idx[0] == 0 and val[0] == -np.inf and flags & orc.FLAG_EMPTY_MASK
    # words past the mask length disallow: only tokens 0..31 are reachable
    mask = np.full((1, 1), -1, np.int32)
    logits, idx, _, _ = orc.lm_head_argmax(0, W, 64, u16(d["x"]), mask=mask, mask_words=1)
    assert idx[0] == int(np.argmax(logits[0, :32]))
    # a shared mask (stride 0) applies to every row
    d2 = synth.head_table(52, 100, 64, 3)
    mask = synth.pack_mask(np.arange(100)[None, :] % 2 == 1)
    logits, idx, _, _ = orc.lm_head_argmax(0, u16(d2["W"]), 64, u16(d2["x"]), mask=mask,
                                           mask_words=mask.shape[1], mask_stride_words=0)
    for m in range(3):
        assert idx[m] == 1 + 2 * int(np.argmax(logits[m, 1::2]))


def test_argmax_negative_zero_equals_zero(orc):
    i, v, f = orc.argmax_masked(np.array([-0.0, 0.0, -1.0]))
    assert i == 0 and f == 0
    i, v, f = orc.argmax_masked(np.array([-1.0, 0.0, -0.0]))
    assert i == 1


# ---------------------------------------------------------------- quantizers

def test_fp8_quantizer_matches_torch_and_bounds(orc):
    W = u16(synth.normal_bf16(synth._gen(61), (64, 256), 0.02))
    W[5] = 0  # zero row
    codes, scale = orc.quantize_fp8(W)
    Wt = torch.tensor(W.view(np.int16)).view(torch.bfloat16).float()
    a = Wt.abs().amax(dim=1)
    s = a / 448.0
    assert np.array_equal(scale, s.numpy())
    nz = a > 0
    ref = (Wt[nz] / s[nz, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes[nz.numpy()], ref)
    assert scale[5] == 0 and np.all(codes[5] == 0)
    # the absmax element of every row encodes to +-448
    wf = orc.bf16_to_f64(W)
    for r in np.nonzero(nz.numpy())[0]:
        j = int(np.argmax(np.abs(wf[r])))
        assert codes[r, j] in (0x7E, 0xFE)
    # round trip: relative 2^-4 for normals, absolute 2^-10 * s below
    deq = e4m3_table()[codes] * scale.astype(np.float64)[:, None]
    q = np.abs(wf) / np.where(scale > 0, scale, 1)[:, None]
    bound = np.where(q >= 2 ** -6, 2 ** -4 * np.abs(wf), 2 ** -10 * scale[:, None])
    assert np.all(np.abs(deq - wf) <= bound + 1e-30)


def load_golden_nvfp4():
    vals = {}
    with open(os.path.join(GOLDEN, "nvfp4_block.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = rest.split()
    return vals


def test_nvfp4_golden_block(orc):
    gold = load_golden_nvfp4()
    w = u16(bf16([float(v) for v in gold["values"]]))[None, :]
    codes, bscale, g = orc.quantize_nvfp4(w)
    assert g == float(gold["global_scale"][0])
    assert list(bscale[0]) == [int(v, 16) for v in gold["block_scales"]]
    assert list(codes[0]) == [int(v, 16) for v in gold["codes"]]


def test_nvfp4_quantizer_bounds(orc):
    W = u16(synth.normal_bf16(synth._gen(71), (48, 320), 0.02))
    codes, bscale, g = orc.quantize_nvfp4(W)
    wf = orc.bf16_to_f64(W)
    A = np.abs(wf).max()
    assert g == np.float32(np.float32(A) / np.float32(2688.0))
    t8 = e4m3_table()
    assert np.all(bscale <= 0x7E)  # positive, finite, <= 448
    blocks = np.abs(wf).reshape(48, 20, 16).max(axis=2)
    r, b = np.unravel_index(np.argmax(blocks), blocks.shape)
    assert bscale[r, b] == 0x7E  # the block holding the global max gets 448
    S = (t8[bscale].astype(np.float32) * np.float32(g)).astype(np.float64)
    deq = independent_dequant(orc, 2, dict(data=codes, block_scale=bscale, global_scale=g), 320)
    Sx = np.repeat(S, 16, axis=1)
    a = np.abs(wf) / Sx
    step = np.where(a <= 2, 0.25, np.where(a <= 4, 0.5, 1.0)) * Sx
    bound = step + np.maximum(0.0, np.abs(wf) - 6 * Sx)
    assert np.all(np.abs(deq - wf) <= bound * (1 + 1e-6))
    z, zb, zg = orc.quantize_nvfp4(np.zeros((2, 32), np.uint16))
    assert zg == 1.0 and np.all(zb == 0) and np.all(z == 0)


# ---------------------------------------------------------------- RoPE / slots / KV

def test_rope_identities(orc):
    rng = np.random.default_rng(5)
    k = rng.standard_normal(128)
    assert np.array_equal(orc.rope_neox(k, 0, 1e6), k)
    r = orc.rope_neox(k, 1234, 1e6)
    assert np.allclose(k[:64] ** 2 + k[64:] ** 2, r[:64] ** 2 + r[64:] ** 2, rtol=1e-12)
    one = orc.rope_neox(k, 1, 1e6)
    rot = np.array([[math.cos(1), -math.sin(1)], [math.sin(1), math.cos(1)]])
    assert np.allclose(rot @ np.array([k[0], k[64]]), [one[0], one[64]], rtol=1e-15)
    assert np.allclose(orc.rope_neox(orc.rope_neox(k, 300, 1e6), 77, 1e6),
                       orc.rope_neox(k, 377, 1e6), rtol=1e-9, atol=1e-12)
    # the last pair turns slowest: theta = pos * base^(-126/128)
    th = 1000 * 1e6 ** (-126 / 128)
    r = orc.rope_neox(k, 1000, 1e6)
    assert np.isclose(r[63], k[63] * math.cos(th) - k[127] * math.sin(th), rtol=1e-12)


def test_slot_golden_cases(orc):
    with open(os.path.join(GOLDEN, "slot_cases.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 8
    for bt, nb, p, want in rows:
        table = [int(v) for v in bt.split(",")]
        assert orc.slot(table, 16, int(nb), int(p)) == int(want), (bt, p)


def test_kv_encode_matches_torch(orc):
    v = u16(synth.normal_bf16(synth._gen(81), (4096,), 3.0))
    vt = torch.tensor(v.view(np.int16)).view(torch.bfloat16).float()
    assert np.array_equal(orc.kv_encode(v, 1.0), vt.to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    assert np.array_equal(orc.kv_encode(v, 0.5), (vt / 0.5).to(torch.float8_e4m3fn).view(torch.uint8).numpy())


def test_prefill_rows_stagewise(orc):
    d = synth.prefill_inputs(seed=91, R=40, vocab=64, h=64, nkv=2, hd=32)
    U = {k: (u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else
             (v.numpy() if isinstance(v, torch.Tensor) else v)) for k, v in d.items()}
    rows = np.array([0, 7, 16, 39])
    out = orc.prefill_rows(U["embed"], U["tokens"], U["hidden"], U["w_norm_embed"],
                           U["w_norm_hidden"], U["eps"], U["fc"], U["wk"], U["wv"], 2, 32,
                           U["rope_base"], U["rope_pos"], 0, U["block_table"], 16,
                           U["num_blocks"], 1.0, 1.0, rows)
    assert out["flags"] == 0
    for i, r in enumerate(rows):
        y, _, _ = orc.combine(U["embed"], U["tokens"][r:r + 1], U["hidden"][r:r + 1],
                              U["w_norm_embed"], U["w_norm_hidden"], U["eps"], U["fc"])
        assert np.array_equal(out["y"][i], y[0])
        yf = orc.bf16_to_f64(y[0])
        k = orc.f64_to_bf16(orc.bf16_to_f64(U["wk"]) @ yf)
        v = orc.f64_to_bf16(orc.bf16_to_f64(U["wv"]) @ yf)
        assert np.array_equal(out["v"][i], v)
        for hh in range(2):
            kr = orc.f64_to_bf16(orc.rope_neox(orc.bf16_to_f64(k[hh * 32:(hh + 1) * 32]),
                                               U["rope_pos"][r], U["rope_base"]))
            assert np.array_equal(out["k_rot"][i, hh * 32:(hh + 1) * 32], kr)
        assert np.array_equal(out["k_codes"][i], orc.kv_encode(out["k_rot"][i], 1.0))
        assert np.array_equal(out["v_codes"][i], orc.kv_encode(v, 1.0))
        assert out["slot"][i] == orc.slot(U["block_table"], 16, U["num_blocks"], r)
    # a cache row past the block table is flagged and not given a slot
    bad = orc.prefill_rows(U["embed"], U["tokens"], U["hidden"], U["w_norm_embed"],
                           U["w_norm_hidden"], U["eps"], U["fc"], U["wk"], U["wv"], 2, 32,
                           U["rope_base"], U["rope_pos"], 10_000, U["block_table"], 16,
                           U["num_blocks"], 1.0, 1.0, rows[:1])
    assert bad["flags"] & orc.FLAG_BAD_SLOT and bad["slot"][0] == -1


def test_head_table_planted_gap_full_size(orc):
    """The benchmark's BF16 table (154,880 x 4,096): the planted row wins by >= 0.5."""
    cfg = synth.BF16_HEAD
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], 1)
    logits, idx, val, _ = orc.lm_head_argmax(0, u16(d["W"]), cfg["K"], u16(d["x"]))
    assert idx[0] == d["top"][0]
    srt = np.sort(logits[0])
    assert srt[-1] - srt[-2] >= 0.5


def test_top1_logprob_pins(orc):
    """Log-softmax at the argmax: closed forms that any mistake in the sum, the mask
    handling or the max subtraction would break."""
    n = 1000
    rng = np.random.default_rng(3)
    for c in (0.0, 3.5, -7.25):  # equal logits: a uniform softmax
        assert orc.top1_logprob(np.full(n, c)) == pytest.approx(-np.log(n), abs=1e-12)
    allowed = rng.choice(n, 37, replace=False)
    mask = np.zeros((n + 31) // 32, np.int32)
    for t in allowed:
        mask[t // 32] |= np.int32(np.uint32(1 << (t % 32)).view(np.int32))
    logits = np.where(np.isin(np.arange(n), allowed), 2.0, 50.0)  # disallowed ones larger
    assert orc.top1_logprob(logits, mask, mask.size) == pytest.approx(-np.log(37), abs=1e-12)
    one = np.zeros_like(mask)
    one[allowed[0] // 32] = np.int32(np.uint32(1 << (allowed[0] % 32)).view(np.int32))
    assert orc.top1_logprob(rng.normal(size=n), one, one.size) == 0.0
    tied = rng.normal(size=n)
    tied[[10, 500]] = 1000.0  # the rest add exp(-1000 + O(1)) = 0 in double
    assert orc.top1_logprob(tied) == pytest.approx(-np.log(2.0), abs=1e-15)
    l = rng.normal(size=n) * 3.0
    assert orc.top1_logprob(l + 123.0) == pytest.approx(orc.top1_logprob(l), abs=1e-12)
    assert orc.top1_logprob(l) < 0.0
    assert orc.top1_logprob(l, np.zeros_like(mask), mask.size) == -np.inf
    # through the sweep: a zero input makes every logit 0
    k = 256
    w = synth.as_u16(synth.normal_bf16(synth._gen(31), (300, k), 0.02))
    lg, idx, _, _ = orc.lm_head_argmax(0, w, k, np.zeros((1, k), np.uint16))
    assert idx[0] == 0 and orc.top1_logprob(lg[0]) == pytest.approx(-np.log(300), abs=1e-12)


def test_fp8_x_two_term_split(orc):
    """The reading behind the tensor-core FP8 sweep: an input row scaled by 2^e (its
    largest |x| in [128, 256)) and split into hi = e4m3(x 2^e), lo = e4m3(x 2^e - hi)
    sums back to x 2^e exactly for every element with |x| >= 2^-9 max|x| (8 significant
    bits = 4 + 4), and within 2^-10 (scaled units, i.e. 2^-17 max|x|) below that."""
    rng = np.random.default_rng(11)
    for scale in (1.0, 3e-3, 7e5, 1e-20):
        v = np.concatenate([rng.standard_normal(3000), rng.standard_normal(500) * 1e-3,
                            rng.standard_normal(500) * 1e-6, [0.0, 1.0, -1.0, 2.0 ** -9]])
        xb = orc.f64_to_bf16(v * scale)
        x = orc.bf16_to_f64(xb)
        a = np.abs(x).max()
        e = 8 - math.frexp(a)[1]
        xs = x * 2.0 ** e
        assert 128 <= np.abs(xs).max() < 256
        hi = orc.e4m3_value(orc.e4m3_encode(xs))
        lo = orc.e4m3_value(orc.e4m3_encode(xs - hi))
        err = np.abs(hi + lo - xs)
        big = np.abs(x) >= 2.0 ** -9 * a
        assert big.sum() > 2900 and np.all(err[big] == 0.0)
        assert np.all(err <= 2.0 ** -10)
        assert np.all(err * 2.0 ** -e <= 2.0 ** -17 * a)
    # the bound is reached: an element whose scaled value sits halfway between two
    # subnormal E4M3 steps keeps half a step
    xs = np.array([200.0, 2.0 ** -10 * 3])
    hi = orc.e4m3_value(orc.e4m3_encode(xs))
    lo = orc.e4m3_value(orc.e4m3_encode(xs - hi))
    assert abs(hi[1] + lo[1] - xs[1]) == 2.0 ** -10


def _six_terms(orc, xs):
    """The six-term split of one scaled input row (per 16-element block: s = 2^se the
    smallest power of two >= max|block| / 4, at least 2^-10; balanced base-8 digits
    d_t = rint(r_t / (s 8^-t)), r_{t+1} = r_t - d_t s 8^-t), written independently of the
    kernel with numpy; returns (digits [6, k], se per block, reconstruction)."""
    k = xs.size
    xb = xs.reshape(-1, 16)
    a = np.abs(xb).max(axis=1)
    se = np.full(a.shape, -10, dtype=np.int64)
    nz = a > 0
    se[nz] = np.maximum(np.ceil(np.log2(a[nz] / 4)).astype(np.int64), -10)
    r = xb.copy()
    digits = np.zeros((6,) + xb.shape)
    rec = np.zeros_like(xb)
    for t in range(6):
        u = np.ldexp(1.0, se - 3 * t)[:, None]
        d = np.rint(r / u)
        digits[t] = d
        rec += d * u
        r = r - d * u
    return digits.reshape(6, k), se, rec.reshape(k)


def test_nvfp4_x_six_term_split(orc):
    """The reading behind the block-scaled NVFP4 sweep: an input row scaled by 2^e (its
    largest |x| in [128, 256)) and written per 16-element block as six E2M1 terms with one
    power-of-two E4M3 scale: every digit d_t lies in [-4, 4] (so d_t / 2 is an E2M1 value),
    the block scale 2 s is an E4M3 value, every element whose binary exponent is within 9
    of its block's largest |x| is represented exactly (its 8 significant bits end at or
    above the last digit's unit s 8^-5 < 2^-16 max), and the rest within 2^-17 of the
    block's largest |x|; where s sits at its 2^-10 floor (blocks below 2^-8 in scaled units)
    every element is within 2^-26 in scaled units instead."""
    rng = np.random.default_rng(12)
    for scale in (1.0, 3e-3, 7e5, 1e-20):
        v = np.concatenate([rng.standard_normal(3008), rng.standard_normal(512) * 1e-3,
                            rng.standard_normal(512) * 1e-6, rng.standard_normal(16) * 1e-30,
                            np.zeros(16), [1.0, -1.0, 2.0 ** -9, 3.0] + [0.0] * 12])
        xb = orc.f64_to_bf16(v * scale)
        x = orc.bf16_to_f64(xb)
        a = np.abs(x).max()
        e = 8 - math.frexp(a)[1]
        xs = x * 2.0 ** e
        assert 128 <= np.abs(xs).max() < 256
        digits, se, rec = _six_terms(orc, xs)
        assert np.all(np.abs(digits) <= 4)
        half = digits / 2
        assert np.array_equal(orc.e2m1_value(orc.e2m1_encode(half)), half)
        sc = np.ldexp(1.0, se + 1)
        assert np.array_equal(orc.e4m3_value(orc.e4m3_encode(sc)), sc)
        err = np.abs(rec - xs)
        bmax = np.repeat(np.abs(xs.reshape(-1, 16)).max(axis=1), 16)
        ex = np.frexp(np.abs(xs))[1]
        bex = np.frexp(bmax)[1]
        floor = np.repeat(se == -10, 16)
        near = (xs != 0) & (bex - ex <= 9) & ~floor
        assert near.sum() > 3500 and np.all(err[near] == 0.0)
        assert np.any(err[(xs != 0) & (bex - ex > 9)] > 0)  # and not beyond
        assert np.all(err[~floor] <= 2.0 ** -17 * bmax[~floor])
        assert np.all(err[floor] <= 2.0 ** -26)
    # the bound is reached: an element 2^-14 below its block's largest, halfway between
    # two steps of the last term, keeps half a step
    xs = np.zeros(16)
    xs[0], xs[1] = 200.0, 2.0 ** -7 * 1.5 + 2.0 ** -12 * 1.5
    _, se, rec = _six_terms(orc, xs)
    assert se[0] == 6 and abs(rec[1] - xs[1]) <= 2.0 ** -17 * 200.0


# ---------------------------------------------------------------- decode attention pins
def _attn_case(orc, seed, nq=8, nkv=2, hd=64, seq=40, bs=16, extra_blocks=3):
    rng = np.random.default_rng(seed)
    nb = seq // bs + 1 + extra_blocks
    bt = rng.permutation(nb).astype(np.int32)
    kc = orc_codes(orc, rng, (nb, bs, nkv, hd))
    vc = orc_codes(orc, rng, (nb, bs, nkv, hd))
    q = orc.f64_to_bf16(rng.normal(0, 1, (nq, hd)))
    return q, kc, vc, bt, nb


def orc_codes(orc, rng, shape):
    # E4M3 codes of N(0, 1) values (finite codes only: the NaN pattern never occurs)
    return orc.e4m3_encode(rng.normal(0, 1, shape)).reshape(shape)


def _dq(orc, codes):
    return orc.e4m3_value(codes.reshape(-1)).reshape(codes.shape)


def test_attn_single_row_returns_its_values(orc):
    q, kc, vc, bt, nb = _attn_case(orc, 1, seq=1)
    out, flags = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 1, k_scale=0.5, v_scale=0.25)
    assert flags == 0
    slot = orc.slot(bt, 16, nb, 0)
    vrow = _dq(orc, vc.reshape(-1, 2, 64)[slot])  # [nkv, hd]
    for i in range(8):
        assert np.array_equal(out[i], 0.25 * vrow[i // 4])  # exact: one weight of 1


def test_attn_zero_scale_and_equal_keys_average_the_values(orc):
    q, kc, vc, bt, nb = _attn_case(orc, 2, seq=40)
    slots = [orc.slot(bt, 16, nb, p) for p in range(40)]
    vrows = _dq(orc, vc.reshape(-1, 2, 64)[slots])  # [seq, nkv, hd]
    mean = vrows.mean(axis=0)
    out, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 40, scale=0.0)
    for i in range(8):
        assert np.allclose(out[i], mean[i // 4], rtol=0, atol=1e-12)
    kc2 = kc.copy().reshape(-1, 2, 64)
    kc2[slots] = kc2[slots[0]]  # every row the same key
    out2, _ = orc.paged_decode_attn(q, 2, kc2.reshape(kc.shape), vc, bt, 16, nb, 40)
    for i in range(8):
        assert np.allclose(out2[i], mean[i // 4], rtol=0, atol=1e-12)


def test_attn_planted_key_dominates_without_overflow(orc):
    q, kc, vc, bt, nb = _attn_case(orc, 3, nq=2, nkv=1, seq=33)
    qv = np.zeros((2, 64))
    qv[:, 0] = 1.0
    q = orc.f64_to_bf16(qv)
    kflat = kc.reshape(-1, 1, 64).copy()
    slots = [orc.slot(bt, 16, nb, p) for p in range(33)]
    kflat[slots] = orc.e4m3_encode(np.zeros(64))
    kflat[slots[17], 0, 0] = orc.e4m3_encode(np.array([448.0]))[0]
    out, _ = orc.paged_decode_attn(q, 1, kflat.reshape(kc.shape), vc, bt, 16, nb, 33, scale=2.0)
    # the planted row scores 896 against 0 for the rest: its weight is 1 - 32 e^-896
    assert np.all(np.isfinite(out))
    want = _dq(orc, vc.reshape(-1, 1, 64)[slots[17], 0])
    assert np.array_equal(out[0], want) and np.array_equal(out[1], want)


def test_attn_block_permutation_and_head_groups(orc):
    q, kc, vc, bt, nb = _attn_case(orc, 4, seq=45)
    out, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 45)
    # move every physical block to a new place and rewrite the block table to match
    perm = np.random.default_rng(9).permutation(nb)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    out2, _ = orc.paged_decode_attn(q, 2, kc2, vc2, perm[bt].astype(np.int32), 16, nb, 45)
    assert np.array_equal(out, out2)
    # query heads 0-3 read kv head 0 and 4-7 kv head 1: head 5 equals a one-group run of
    # kv head 1 alone
    out1, _ = orc.paged_decode_attn(q[5:6], 1, np.ascontiguousarray(kc[:, :, 1:2]),
                                    np.ascontiguousarray(vc[:, :, 1:2]), bt, 16, nb, 45)
    assert np.array_equal(out[5], out1[0])


def test_attn_missing_block_flags_and_skips(orc):
    q, kc, vc, bt, nb = _attn_case(orc, 5, seq=40)
    out, flags = orc.paged_decode_attn(q, 2, kc, vc, bt[:2], 16, nb, 40)  # rows 32.. have no block
    assert flags & orc.FLAG_BAD_SLOT
    ref, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 32)
    assert np.array_equal(out, ref)



# ---------------------------------------------------------------- norm mode and k norm pins
def test_one_plus_w_mode_is_plain_mode_on_shifted_weights(orc):
    """norm_mode 1 multiplies by 1 + w: with w = 0 it is plain mode with unit weights, and
    with weights whose 1 + w is a bf16 value it is plain mode with those values."""
    rng = np.random.default_rng(31)
    x = orc.f64_to_bf16(rng.normal(0, 1, 64))
    zero = np.zeros(64, np.uint16)
    one = orc.f64_to_bf16(np.ones(64))
    assert np.array_equal(orc.rmsnorm(x, zero, 1e-6, norm_mode=1), orc.rmsnorm(x, one, 1e-6))
    w = rng.choice([0.0, 0.5, -0.25, 0.125, 1.0, -0.5], 64)
    assert np.array_equal(orc.rmsnorm(x, orc.f64_to_bf16(w), 1e-6, norm_mode=1),
                          orc.rmsnorm(x, orc.f64_to_bf16(1.0 + w), 1e-6))
    d = synth.tiny_draft(seed=5, vocab=50, h=32, M=2)
    u = synth.as_u16
    y1, c1, _ = orc.combine(u(d["embed"]), d["tokens"].numpy(), u(d["hidden"]), zero[:32],
                            zero[:32], 1e-6, u(d["fc"]), norm_mode=1)
    y0, c0, _ = orc.combine(u(d["embed"]), d["tokens"].numpy(), u(d["hidden"]), one[:32],
                            one[:32], 1e-6, u(d["fc"]))
    assert np.array_equal(c1, c0) and np.array_equal(y1, y0)


def _kn_case(orc, seed, k_norm, pos0=0, norm_mode=0, same_rows=False, norm_w=None):
    d = synth.prefill_inputs(seed=seed, R=6, vocab=40, h=256, nkv=2, hd=64)
    if norm_w is not None:  # both combiner norm weights set to this constant
        d["w_norm_embed"] = torch.full((256,), norm_w, dtype=torch.bfloat16)
        d["w_norm_hidden"] = torch.full((256,), norm_w, dtype=torch.bfloat16)
    if same_rows:  # every row of a head's Wk the same: each k head is a constant vector
        wk = d["wk"].clone()
        for hh in range(2):
            wk[hh * 64:(hh + 1) * 64] = wk[hh * 64]
        d["wk"] = wk
    d["rope_pos"] = torch.full((6,), pos0, dtype=torch.int32)
    U = {k: (synth.as_u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else
             (v.numpy() if isinstance(v, torch.Tensor) else v)) for k, v in d.items()}
    out = orc.prefill_rows(U["embed"], U["tokens"], U["hidden"], U["w_norm_embed"],
                           U["w_norm_hidden"], U["eps"], U["fc"], U["wk"], U["wv"], 2, 64,
                           U["rope_base"], U["rope_pos"], 0, U["block_table"], 16,
                           U["num_blocks"], 1.0, 1.0, np.arange(6), norm_mode=norm_mode,
                           k_norm=k_norm)
    return out, U


def test_k_norm_constant_head_closed_form(orc):
    """A head whose Wk rows are all equal gives k = c 1; its k norm at RoPE position 0 (the
    identity) is bf16(c / sqrt(c^2 + eps) w_j)."""
    rng = np.random.default_rng(32)
    w = orc.f64_to_bf16(rng.normal(1.0, 0.1, 64))
    plain, _ = _kn_case(orc, 41, None, same_rows=True)
    normed, U = _kn_case(orc, 41, w, same_rows=True)
    c = bf16_to_f64_(plain["k_rot"].reshape(6, 2, 64)[:, :, 0])  # pos 0: k itself
    want = orc.f64_to_bf16(c[:, :, None] / np.sqrt(c[:, :, None] ** 2 + U["eps"])
                           * bf16_to_f64_(w)[None, None, :])
    assert np.array_equal(normed["k_rot"].reshape(6, 2, 64), want)
    assert np.array_equal(normed["v"], plain["v"])  # v is untouched


def test_k_norm_unit_rms_and_mode(orc):
    """With unit weights every k head has RMS 1 before RoPE; RoPE keeps pair norms, so the
    stored head's RMS stays 1 up to bf16 rounding. Mode 1 with w = 0 equals unit weights."""
    ones = orc.f64_to_bf16(np.ones(64))
    out, _ = _kn_case(orc, 42, ones, pos0=100)
    k = bf16_to_f64_(out["k_rot"]).reshape(6, 2, 64)
    rms = np.sqrt((k ** 2).mean(axis=2))
    assert np.all(np.abs(rms - 1.0) < 5e-3), rms
    # mode 1 applies 1 + w to every norm of the call: zero weights there are unit weights
    out0, _ = _kn_case(orc, 42, ones, pos0=100, norm_w=1.0)
    out1, _ = _kn_case(orc, 42, np.zeros(64, np.uint16), pos0=100, norm_mode=1, norm_w=0.0)
    assert np.array_equal(out1["k_rot"], out0["k_rot"]) and np.array_equal(out1["v"], out0["v"])


def bf16_to_f64_(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_k_norm_comes_before_rope(orc):
    """A constant head k = c 1 with non-uniform k-norm weights w at RoPE position 37: the
    normed head bf16(s w), s = c / sqrt(c^2 + eps), rotated by RoPE (pinned above), then
    rounded -- which fixes the order (rotating first and normalizing after differs)."""
    rng = np.random.default_rng(33)
    w = orc.f64_to_bf16(rng.normal(1.0, 0.3, 64))
    plain, _ = _kn_case(orc, 41, None, same_rows=True)  # position 0: k itself
    normed, U = _kn_case(orc, 41, w, pos0=37, same_rows=True)
    c = bf16_to_f64_(plain["k_rot"].reshape(6, 2, 64)[:, :, 0])
    got = normed["k_rot"].reshape(6, 2, 64)
    for r in range(6):
        for hh in range(2):
            s = c[r, hh] / np.sqrt(c[r, hh] ** 2 + U["eps"])
            kn = bf16_to_f64_(orc.f64_to_bf16(s * bf16_to_f64_(w)))
            want = orc.f64_to_bf16(orc.rope_neox(kn, 37.0, U["rope_base"]))
            assert np.array_equal(got[r, hh], want), (r, hh)


# ---------------------------------------------------------------- input norm (normed2) pins
def _in_case(orc, seed, in_norm, norm_mode=0, fc_scale=1.0, eps=None, onehot_v=False):
    d = synth.prefill_inputs(seed=seed, R=5, vocab=40, h=256, nkv=2, hd=64)
    if fc_scale != 1.0:
        d["fc"] = (d["fc"].float() * fc_scale).to(torch.bfloat16)
    if eps is not None:
        d["eps"] = eps
    if onehot_v:  # row i of Wv selects element (7 i + 3) mod h
        wv = torch.zeros_like(d["wv"])
        for i in range(wv.shape[0]):
            wv[i, (7 * i + 3) % 256] = 1.0
        d["wv"] = wv
    U = {k: (synth.as_u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else
             (v.numpy() if isinstance(v, torch.Tensor) else v)) for k, v in d.items()}
    out = orc.prefill_rows(U["embed"], U["tokens"], U["hidden"], U["w_norm_embed"],
                           U["w_norm_hidden"], U["eps"], U["fc"], U["wk"], U["wv"], 2, 64,
                           U["rope_base"], U["rope_pos"], 0, U["block_table"], 16,
                           U["num_blocks"], 1.0, 1.0, np.arange(5), norm_mode=norm_mode,
                           in_norm=in_norm)
    return out, U


def test_in_norm_feeds_k_and_v_through_the_pinned_rmsnorm(orc):
    """One-hot Wv rows read single elements of k/v's input: with the input norm that input is
    the (separately pinned) RMSNorm of the stored fc output y, in both weight modes."""
    rng = np.random.default_rng(35)
    w = orc.f64_to_bf16(rng.normal(0.5, 0.4, 256))
    for mode in (0, 1):
        out, U = _in_case(orc, 51, w, norm_mode=mode, onehot_v=True)
        for r in range(5):
            n2 = orc.rmsnorm(out["y"][r], w, U["eps"], norm_mode=mode)
            want = n2[(7 * np.arange(128) + 3) % 256]
            assert np.array_equal(out["v"][r], want), (mode, r)
    plain, _ = _in_case(orc, 51, None, onehot_v=True)
    assert np.array_equal(plain["v"][0], plain["y"][0][(7 * np.arange(128) + 3) % 256])


def test_in_norm_zero_weights_and_scale_invariance(orc):
    """Zero input-norm weights (plain mode) zero k and v. With eps = 0, doubling fc doubles
    y exactly; the normed input, hence k and v, stay bit-identical -- and without the input
    norm v doubles exactly, so the invariance is the norm's."""
    zero = np.zeros(256, np.uint16)
    out, _ = _in_case(orc, 52, zero)
    assert np.all(bf16_to_f64_(out["k_rot"]) == 0) and np.all(bf16_to_f64_(out["v"]) == 0)
    w = orc.f64_to_bf16(np.random.default_rng(36).normal(1.0, 0.2, 256))
    a, _ = _in_case(orc, 53, w, eps=0.0)
    b, _ = _in_case(orc, 53, w, eps=0.0, fc_scale=2.0)
    assert np.array_equal(bf16_to_f64_(b["y"]), 2 * bf16_to_f64_(a["y"]))
    assert np.array_equal(a["k_rot"], b["k_rot"]) and np.array_equal(a["v"], b["v"])
    pa, _ = _in_case(orc, 53, None, eps=0.0)
    pb, _ = _in_case(orc, 53, None, eps=0.0, fc_scale=2.0)
    assert np.array_equal(bf16_to_f64_(pb["v"]), 2 * bf16_to_f64_(pa["v"]))
