"""The drafter-context prefill on the GPU against the oracle.

Stage by stage: the tcgen05 GEMM (one-hot rows select B rows exactly; random operands
within 2e-2 + 1e-2|ref|), the E4M3 encode + paged scatter given the same bf16 k'/v
(bit-exact codes and slots, every other cache byte untouched), then the whole prefill
on a small multi-chunk prompt (every row) and on the benchmark prompt (32,768 rows,
hidden 5,120, chunks of 2,048; sampled rows spread over all chunks).

End to end the codes are not bit-exact by construction: the GPU accumulates the two
projections in fp32 and the oracle in fp64, so bf16(y) and bf16(k) can differ by an
ulp, which the RoPE rotation and the E4M3 rounding can expose. The criterion is the
activation tolerance carried through: RoPE rotates each pair (k_j, k_{j+hd/2}) without
changing its norm, so a k' value may differ from the oracle's by 2e-2 + 1e-2 x the pair
norm, plus one E4M3 step of the final rounding (where the rotation nearly cancels, a
tiny k' inherits the absolute error of inputs near the pair norm); a v value by
2e-2 + 1e-2 |v| plus one step. At least 98% of codes are identical; slots are exact.
"""
import numpy as np
import pytest
import torch

from helpers import assert_close, bf16_bits_to_f64, to_dev, to_dev_u16, u16_of
from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu

SENTINEL = 0x7F  # E4M3 NaN: never produced by a saturating encode


def gemm(A, B):
    M, K = A.shape
    N = B.shape[0]
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    L.mtp_debug_gemm_bf16(to_dev_u16(A), to_dev_u16(B), C, M, N, K)
    torch.cuda.synchronize()
    return u16_of(C)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 512, 640), (1000, 1024, 4096),
                                   (1400, 768, 512),    # 11 row blocks: the last pair has one
                                   (2048, 4096, 256)])  # the last: several tiles per SM pair
def test_gemm_matches_numpy(orc, M, N, K):
    A = synth.as_u16(synth.normal_bf16(synth._gen(M + N), (M, K), 1.0))
    B = synth.as_u16(synth.normal_bf16(synth._gen(K + 3), (N, K), 0.02))
    C = gemm(A, B)
    ref = orc.bf16_to_f64(A) @ orc.bf16_to_f64(B).T
    assert_close(bf16_bits_to_f64(C), ref, "C")


def test_gemm_one_hot_rows_are_exact(orc):
    M, N, K = 256, 512, 1024
    B = synth.as_u16(synth.normal_bf16(synth._gen(5), (N, K), 1.0))
    A = np.zeros((M, K), np.uint16)
    cols = (np.arange(M) * 37) % K
    A[np.arange(M), cols] = 0x3F80  # 1.0
    C = gemm(A, B)
    assert np.array_equal(C, B[:, cols].T)


def kv_ordinal(c):
    c = np.asarray(c, np.int32)
    return np.where(c & 0x80, -(c & 0x7F), c & 0x7F)


def new_caches(num_blocks, bs, nkv, hd):
    k = torch.full((num_blocks, bs, nkv, hd), SENTINEL, dtype=torch.uint8, device="cuda")
    v = torch.full((num_blocks, bs, nkv, hd), SENTINEL, dtype=torch.uint8, device="cuda")
    return k, v


def test_kv_write_stage_bit_exact(orc):
    R, nkv, hd, bs = 200, 2, 128, 16
    nb = R // bs + 3
    table = torch.randperm(nb, generator=synth._gen(4)).to(torch.int32)
    k_rot = synth.as_u16(synth.normal_bf16(synth._gen(6), (R, nkv * hd), 2.0))
    v = synth.as_u16(synth.normal_bf16(synth._gen(7), (R, nkv * hd), 2.0))
    for start, ks, vs in ((0, 1.0, 1.0), (5, 0.5, 2.0)):
        kc, vc = new_caches(nb, bs, nkv, hd)
        err = torch.zeros((1,), dtype=torch.int32, device="cuda")
        L.mtp_debug_kv_write(to_dev_u16(k_rot), to_dev_u16(v), R, nkv, hd, start,
                             table.cuda(), nb, bs, nb, kc, vc, ks, vs, err)
        torch.cuda.synchronize()
        kc = kc.cpu().numpy().reshape(-1, nkv * hd)
        vc = vc.cpu().numpy().reshape(-1, nkv * hd)
        written = np.zeros(kc.shape[0], bool)
        for r in range(R):
            slot = orc.slot(table.numpy(), bs, nb, start + r)
            if slot < 0:
                continue
            written[slot] = True
            assert np.array_equal(kc[slot], orc.kv_encode(k_rot[r], ks)), r
            assert np.array_equal(vc[slot], orc.kv_encode(v[r], vs)), r
        assert np.all(kc[~written] == SENTINEL) and np.all(vc[~written] == SENTINEL)
        expect_bad = any(orc.slot(table.numpy(), bs, nb, start + r) < 0 for r in range(R))
        assert bool(err.item() & L.MTP_DEVFLAG_BAD_SLOT) == expect_bad


def run_prefill(d, chunk, extra_blocks_cache=0):
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    nb = int(d["num_blocks"]) + extra_blocks_cache
    kc, vc = new_caches(nb, d["block_size"], d["nkv"], d["hd"])
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    api.prefill_kv(dev, kc, vc, chunk_rows=chunk, dev_err=err)
    torch.cuda.synchronize()
    return kc.cpu().numpy(), vc.cpu().numpy(), int(err.item())


def oracle_rows(orc, d, rows):
    U = {k: (synth.as_u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else
             (v.numpy() if isinstance(v, torch.Tensor) else v)) for k, v in d.items()}
    return orc.prefill_rows(U["embed"], U["tokens"], U["hidden"], U["w_norm_embed"],
                            U["w_norm_hidden"], U["eps"], U["fc"], U["wk"], U["wv"], d["nkv"],
                            d["hd"], d["rope_base"], U["rope_pos"], d["cache_start"],
                            U["block_table"], d["block_size"], d["num_blocks"], d["k_scale"],
                            d["v_scale"], rows, norm_mode=int(d.get("norm_mode", 0)),
                            k_norm=U.get("k_norm"), in_norm=U.get("in_norm"))


def e4m3_step(v):
    """Spacing of E4M3 values at |v| (2^-9 below the smallest normal)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))


def check_rows(orc, d, kc, vc, rows, min_exact=0.98):
    ref = oracle_rows(orc, d, rows)
    nkv, hd = d["nkv"], d["hd"]
    kc = kc.reshape(-1, nkv * hd)
    vc = vc.reshape(-1, nkv * hd)
    exact = total = 0
    for i, r in enumerate(rows):
        slot = ref["slot"][i]
        assert slot >= 0
        kr = bf16_bits_to_f64(ref["k_rot"][i]).reshape(nkv, 2, hd // 2)
        pair = np.sqrt((kr ** 2).sum(axis=1, keepdims=True))
        k_scale = np.broadcast_to(pair, kr.shape).reshape(-1) / d["k_scale"]
        v_scale = np.abs(bf16_bits_to_f64(ref["v"][i])) / d["v_scale"]
        for got, want, sc in ((kc[slot], ref["k_codes"][i], k_scale),
                              (vc[slot], ref["v_codes"][i], v_scale)):
            gv, wv = orc.e4m3_value(got), orc.e4m3_value(want)
            lim = np.maximum(e4m3_step(gv), e4m3_step(wv)) + 2e-2 + 1e-2 * sc
            bad = np.abs(gv - wv) > lim
            assert not bad.any(), (r, np.nonzero(bad)[0][:5], got[bad][:5], want[bad][:5])
            exact += int((got == want).sum())
            total += got.size
    assert exact / total >= min_exact, exact / total
    return exact / total


def test_prefill_small_multi_chunk(orc):
    d = synth.prefill_inputs(seed=77, R=300, vocab=500, h=256, nkv=2, hd=128)
    kc, vc, err = run_prefill(d, chunk=128)
    assert err == 0
    check_rows(orc, d, kc, vc, np.arange(300))
    # every cache row that no prompt row maps to keeps the sentinel
    slots = {orc.slot(d["block_table"].numpy(), 16, d["num_blocks"], r) for r in range(300)}
    flat = kc.reshape(-1, 256)
    untouched = [s for s in range(flat.shape[0]) if s not in slots]
    assert np.all(flat[untouched] == SENTINEL)


def test_prefill_other_heads_and_positions(orc):
    d = synth.prefill_inputs(seed=78, R=70, vocab=300, h=512, nkv=4, hd=64)
    d["rope_pos"] = torch.arange(1000, 1070, dtype=torch.int32)
    d["cache_start"] = 5
    d["num_blocks"] = int(d["num_blocks"]) + 1
    d["block_table"] = torch.randperm(d["num_blocks"], generator=synth._gen(3)).to(torch.int32)
    kc, vc, err = run_prefill(d, chunk=64)
    assert err == 0
    check_rows(orc, d, kc, vc, np.arange(70))


@pytest.mark.parametrize("mode", [0, 1])
def test_prefill_k_norm_and_one_plus_w(orc, mode):
    """A per-head k norm before RoPE, with plain and 1 + w norm weights."""
    d = synth.prefill_inputs(seed=84 + mode, R=150, vocab=300, h=256, nkv=2, hd=128)
    g = synth._gen(12 + mode)
    d["k_norm"] = synth.normal_bf16(g, (128,), 0.3, mean=0.0 if mode else 1.0)
    d["norm_mode"] = mode
    kc, vc, err = run_prefill(d, chunk=64)
    assert err == 0
    check_rows(orc, d, kc, vc, np.arange(150))
    # the k norm changes the keys: without it the K codes differ
    d0 = dict(d)
    del d0["k_norm"]
    kc0, _, _ = run_prefill(d0, chunk=64)
    assert (kc0 != kc).mean() > 0.3


@pytest.mark.parametrize("mode,k_norm", [(0, False), (1, True)])
def test_prefill_input_norm(orc, mode, k_norm):
    """The input norm between fc and k/v (done in place by each row block's last fc tile):
    three chunks (the last ragged), two fc column tiles per row block, with and without
    the k norm."""
    d = synth.prefill_inputs(seed=86 + mode, R=300, vocab=300, h=512, nkv=2, hd=128)
    g = synth._gen(14 + mode)
    d["in_norm"] = synth.normal_bf16(g, (512,), 0.3, mean=0.0 if mode else 1.0)
    if k_norm:
        d["k_norm"] = synth.normal_bf16(g, (128,), 0.3, mean=0.0 if mode else 1.0)
    d["norm_mode"] = mode
    kc, vc, err = run_prefill(d, chunk=128)
    assert err == 0
    check_rows(orc, d, kc, vc, np.arange(300))
    d0 = dict(d)
    del d0["in_norm"]
    _, vc0, _ = run_prefill(d0, chunk=128)
    assert (vc0 != vc).mean() > 0.3


def test_prefill_bad_slot_and_token_flags(orc):
    d = synth.prefill_inputs(seed=79, R=40, vocab=100, h=256, nkv=2, hd=128)
    d["tokens"] = d["tokens"].clone()
    d["tokens"][3] = 1000
    d["block_table"] = d["block_table"][:2].clone()  # rows 32.. have no block
    kc, vc, err = run_prefill(d, chunk=64)
    assert err & L.MTP_DEVFLAG_BAD_SLOT and err & L.MTP_DEVFLAG_BAD_TOKEN
    check_rows(orc, d, kc, vc, np.arange(32))


def test_prefill_full_prompt_sampled_rows(orc):
    d = synth.prefill_inputs()
    kc, vc, err = run_prefill(d, chunk=synth.PREFILL["chunk"])
    assert err == 0
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([
        [0, 1, 2047, 2048, 32767],
        rng.choice(d["R"], 59, replace=False)]))
    frac = check_rows(orc, d, kc, vc, rows)
    print(f"prefill 32,768 rows: {frac:.4%} of sampled codes identical to the oracle's")


def test_prefill_lanes_and_graph_capture_agree(orc):
    """The whole call is one kernel on the caller's stream. Two workspace lanes
    (consecutive chunks overlapping), one lane (chunks ordered through the same buffers),
    the two-lane call on a side stream and a CUDA-graph capture of it write the same cache
    bytes; the rows match the oracle."""
    d = synth.prefill_inputs(seed=81, R=700, vocab=500, h=256, nkv=2, hd=128)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    nb, chunk = int(d["num_blocks"]), 128
    full = L.mtp_prefill_ws_bytes(chunk, 256, 2, 128)
    outs = []
    for nbytes in (full, full // 2):
        kc, vc = new_caches(nb, 16, 2, 128)
        ws = api.aligned_empty(nbytes, 1024, "cuda")
        api.prefill_kv(dev, kc, vc, chunk_rows=chunk, ws=ws)
        torch.cuda.synchronize()
        outs.append((kc.cpu().numpy(), vc.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    kc, vc = new_caches(nb, 16, 2, 128)
    ws = api.aligned_empty(full, 1024, "cuda")
    with torch.cuda.stream(s):
        api.prefill_kv(dev, kc, vc, chunk_rows=chunk, ws=ws)
    s.synchronize()
    assert np.array_equal(kc.cpu().numpy(), outs[0][0])
    kc, vc = new_caches(nb, 16, 2, 128)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            api.prefill_kv(dev, kc, vc, chunk_rows=chunk, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), outs[0][0])
    assert np.array_equal(vc.cpu().numpy(), outs[0][1])
    check_rows(orc, d, outs[0][0], outs[0][1], np.arange(0, 700, 7))


def test_prefill_many_tiles_per_sm(orc):
    """More tiles than SMs (hidden 1,024, 8 KV heads x 128, chunks of 256 rows: 208 tiles),
    so every SM runs several prologue, fc and k/v tiles back to back; both lane counts."""
    d = synth.prefill_inputs(seed=83, R=2048, vocab=900, h=1024, nkv=8, hd=128)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    nb = int(d["num_blocks"])
    full = L.mtp_prefill_ws_bytes(256, 1024, 8, 128)
    outs = []
    for nbytes in (full, full // 2):
        kc, vc = new_caches(nb, 16, 8, 128)
        err = torch.zeros((1,), dtype=torch.int32, device="cuda")
        ws = api.aligned_empty(nbytes, 1024, "cuda")
        api.prefill_kv(dev, kc, vc, chunk_rows=256, ws=ws, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        outs.append((kc.cpu().numpy(), vc.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    rows = np.unique(np.concatenate([[0, 255, 256, 2047],
                                     np.random.default_rng(6).choice(2048, 40, replace=False)]))
    check_rows(orc, d, outs[0][0], outs[0][1], rows)


def test_prefill_odd_row_blocks(orc):
    """Chunks of three 128-row blocks (384 rows; the last chunk 232 rows, two blocks): the
    last 256-row pair block of a full chunk has rows for one CTA of the pair only."""
    d = synth.prefill_inputs(seed=95, R=1000, vocab=400, h=512, nkv=2, hd=128)
    kc, vc, err = run_prefill(d, chunk=384)
    assert err == 0
    check_rows(orc, d, kc, vc, np.arange(1000))


def test_prefill_ragged_chunks_and_one_row(orc):
    """A last chunk of a single row, a chunk that is not a multiple of 128 rows, and a
    one-row prompt."""
    for R, chunk in ((257, 128), (200, 72), (1, 2048)):
        d = synth.prefill_inputs(seed=90 + R, R=R, vocab=400, h=256, nkv=2, hd=128)
        kc, vc, err = run_prefill(d, chunk=chunk)
        assert err == 0
        check_rows(orc, d, kc, vc, np.arange(R))
