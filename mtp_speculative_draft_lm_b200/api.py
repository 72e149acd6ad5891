"""Torch-facing helpers over the C ABI: they allocate device buffers with torch
(memory and streams are torch's job here) and call the ``mtp_*`` entry points.
No arithmetic of the method happens in Python."""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import _lib as L


def _u16(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype in (torch.bfloat16, torch.int16, torch.uint16)
    return t


@dataclass
class Table:
    """A [n, k] weight table on the device in one of the three formats."""
    fmt: int
    n: int
    k: int
    data: torch.Tensor
    row_scale: torch.Tensor | None = None
    block_scale: torch.Tensor | None = None
    global_scale: torch.Tensor | None = None
    desc: L.mtp_weight = field(init=False)

    def __post_init__(self):
        self.desc = L.weight(self.fmt, self.n, self.k, self.data, self.row_scale,
                             self.block_scale, self.global_scale)

    def nbytes(self) -> int:
        b = self.data.numel() * self.data.element_size()
        for t in (self.row_scale, self.block_scale, self.global_scale):
            if t is not None:
                b += t.numel() * t.element_size()
        return b


def bf16_table(w: torch.Tensor) -> Table:
    n, k = w.shape
    return Table(L.MTP_FMT_BF16, n, k, _u16(w.contiguous()))


def quantize_fp8(w: torch.Tensor, stream=None) -> Table:
    n, k = w.shape
    codes = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    scale = torch.empty((n,), dtype=torch.float32, device=w.device)
    L.mtp_quantize_fp8(w, n, k, codes, scale, stream)
    return Table(L.MTP_FMT_FP8_ROW, n, k, codes, row_scale=scale)


def quantize_nvfp4(w: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> Table:
    n, k = w.shape
    codes = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    bscale = torch.empty((n, L.mtp_nvfp4_scale_pitch(k)), dtype=torch.uint8, device=w.device)
    g = torch.empty((1,), dtype=torch.float32, device=w.device)
    nbytes = L.mtp_quantize_nvfp4_ws_bytes(n, k)
    if ws is None:
        ws = torch.zeros((nbytes,), dtype=torch.uint8, device=w.device)
    L.mtp_quantize_nvfp4(w, n, k, codes, bscale, g, ws, ws.numel(), stream)
    return Table(L.MTP_FMT_NVFP4, n, k, codes, block_scale=bscale, global_scale=g)


class LmHead:
    """The fused sweep + argmax over a table, with its zeroed workspace."""

    def __init__(self, table: Table, n_eff: int | None = None, max_m: int = 32):
        self.table = table
        self.n_eff = table.n if n_eff is None else int(n_eff)
        dev = table.data.device
        # room for the host-input entry point's copy of x as well
        nbytes = L.mtp_lm_head_host_ws_bytes(table.desc, self.n_eff, max_m)
        self.ws = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
        self.dev_err = torch.zeros((1,), dtype=torch.int32, device=dev)

    def bytes_per_call(self, M: int, mask_words: int = 0, rows: int | None = None) -> int:
        """Algorithmic bytes of one sweep: the table rows it must read (all n_eff rows, or
        `rows` of them under a grammar mask), the inputs, the mask words and the
        outputs."""
        t = self.table
        frac = (self.n_eff if rows is None else rows) / t.n
        return int(t.nbytes() * frac) + M * t.k * 2 + mask_words * 4 + M * 8

    def __call__(self, x: torch.Tensor, out_idx: torch.Tensor, out_val=None, out_logits=None,
                 mask=None, mask_words=0, mask_stride_words=0, stream=None, out_logprob=None):
        M = x.shape[0]
        if out_logprob is None:
            L.mtp_lm_head_argmax(self.table.desc, self.n_eff, x, M, mask, mask_words,
                                 mask_stride_words, out_idx, out_val, out_logits, self.dev_err,
                                 self.ws, self.ws.numel(), stream)
        else:
            L.mtp_lm_head_argmax_lp(self.table.desc, self.n_eff, x, M, mask, mask_words,
                                    mask_stride_words, out_idx, out_val, out_logprob,
                                    out_logits, self.dev_err, self.ws, self.ws.numel(), stream)

    def argmax_host(self, x_host: torch.Tensor, out_host: torch.Tensor, mask=None, mask_words=0,
                    mask_stride_words=0, stream=None):
        """One draft step from pinned host memory to pinned host memory: x_host bf16
        [M, k] pinned; out_host int32 [2M] pinned receives the indices, then the values
        (float32 bits). Valid once the stream has synchronised."""
        M = x_host.shape[0]
        L.mtp_lm_head_argmax_host(self.table.desc, self.n_eff, x_host, M, mask, mask_words,
                                  mask_stride_words, out_host, self.dev_err, self.ws,
                                  self.ws.numel(), stream)

    def argmax(self, x: torch.Tensor, mask=None, mask_words=0, mask_stride_words=0,
               logits=False, stream=None, logprob=False):
        """Returns (idx, val, logits or None), plus the top-1 log-probabilities when
        logprob is true."""
        M = x.shape[0]
        dev = x.device
        idx = torch.empty((M,), dtype=torch.int32, device=dev)
        val = torch.empty((M,), dtype=torch.float32, device=dev)
        lg = torch.empty((M, self.n_eff), dtype=torch.bfloat16, device=dev) if logits else None
        lp = torch.empty((M,), dtype=torch.float32, device=dev) if logprob else None
        self(x, idx, val, lg, mask, mask_words, mask_stride_words, stream, out_logprob=lp)
        return (idx, val, lg, lp) if logprob else (idx, val, lg)


def table_rows(table: Table, r0: int, r1: int) -> Table:
    """Rows [r0, r1) of a table as a table of its own (views: rows are contiguous, so a
    vocab shard is a base-pointer offset and a smaller n)."""
    rs = table.row_scale[r0:r1] if table.row_scale is not None else None
    bs = table.block_scale[r0:r1] if table.block_scale is not None else None
    return Table(table.fmt, r1 - r0, table.k, table.data[r0:r1], row_scale=rs, block_scale=bs,
                 global_scale=table.global_scale)


def shard_range(n: int, world: int, rank: int, align: int = 16) -> tuple[int, int]:
    """(row_offset, rows) of rank's vocab shard: equal contiguous ranges in units of
    `align` rows (the sweep's 16-row tiles), the last one shorter; empty when there are
    more ranks than units."""
    units = -(-n // align)
    per = -(-units // world) * align
    off = min(n, rank * per)
    return off, min(n, off + per) - off


#: a shard partial: {f32 max logit, i32 global row (INT32_MAX: none allowed), f32 sum of
#: exp(l - max), unused}, stored as 4 float32 words per input row
EMPTY_PARTIAL = (float("-inf"), 2147483647, 0.0)


def exchange_partials(local: torch.Tensor, group=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """All-gathers every rank's [M, 4] partials into [world, M, 4] (rank-major), the one
    collective of the vocab-sharded sweep (NCCL over NVLink on GPUs)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if out is None:
        out = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
    # gathered along dim 0 ([world * M, 4]); viewed back as [world, M, 4]
    flat = out.view((world * local.shape[0],) + tuple(local.shape[1:]))
    dist.all_gather_into_tensor(flat, local.contiguous(), group=group)
    return out


class ShardedLmHead:
    """The lm_head sweep + argmax split by vocab over the ranks of a process group: each
    rank sweeps its own rows (mtp_lm_head_shard_partial), the 16-byte partials are
    all-gathered, and every rank merges them (mtp_argmax_merge_partials)."""

    def __init__(self, shard: Table | None, row_offset: int, group=None, max_m: int = 32):
        self.shard = shard
        self.row_offset = int(row_offset)
        self.group = group
        self.head = LmHead(shard, max_m=max_m) if shard is not None and shard.n > 0 else None
        self._bufs = {}

    def _buffers(self, M: int, dev):
        import torch.distributed as dist

        if M not in self._bufs:
            world = dist.get_world_size(self.group)
            self._bufs[M] = dict(
                local=torch.empty((M, 4), dtype=torch.float32, device=dev),
                parts=torch.empty((world, M, 4), dtype=torch.float32, device=dev),
                idx=torch.empty((M,), dtype=torch.int32, device=dev),
                val=torch.empty((M,), dtype=torch.float32, device=dev),
                lp=torch.empty((M,), dtype=torch.float32, device=dev),
                err=torch.zeros((1,), dtype=torch.int32, device=dev), world=world)
        return self._bufs[M]

    def argmax(self, x: torch.Tensor, mask=None, mask_words=0, mask_stride_words=0,
               logprob=False, stream=None):
        """Returns (idx, val, err) or (idx, val, logprob, err): the merged result, the
        same on every rank; err is the merge's device error word. The returned tensors
        are reused by the next call with the same M."""
        M = x.shape[0]
        b = self._buffers(M, x.device)
        local = b["local"]
        if self.head is None:  # no rows here: an empty partial
            local.zero_()
            local[:, 0] = EMPTY_PARTIAL[0]
            local.view(torch.int32)[:, 1] = EMPTY_PARTIAL[1]
        else:
            L.mtp_lm_head_shard_partial(self.shard.desc, self.shard.n, self.row_offset, x, M, mask,
                                        mask_words, mask_stride_words, local, None,
                                        self.head.dev_err, self.head.ws, self.head.ws.numel(),
                                        stream)
        exchange_partials(local, self.group, out=b["parts"])
        b["err"].zero_()
        lp = b["lp"] if logprob else None
        L.mtp_argmax_merge_partials(b["parts"], b["world"], M, b["idx"], b["val"], lp, b["err"],
                                    stream)
        return (b["idx"], b["val"], lp, b["err"]) if logprob else (b["idx"], b["val"], b["err"])


def combine(embed, token_ids, hidden, w_norm_embed, w_norm_hidden, eps, fc: Table,
            out=None, dev_err=None, stream=None, norm_mode=L.MTP_NORM_W):
    M, h = hidden.shape
    if out is None:
        out = torch.empty((M, h), dtype=torch.bfloat16, device=hidden.device)
    L.mtp_combine(embed, embed.shape[0], token_ids, hidden, M, h, w_norm_embed, w_norm_hidden,
                  eps, norm_mode, fc.desc, out, dev_err, stream)
    return out


def draft_step(embed, token_ids, hidden, w_norm_embed, w_norm_hidden, eps, fc, head,
               n_eff=None, mask=None, mask_words=0, mask_stride_words=0, out_y=None,
               out_idx=None, out_val=None, dev_err=None, stream=None, norm_mode=L.MTP_NORM_W):
    """One whole draft step (combiner + lm_head sweep + argmax) for a small BF16 head in
    one launch: returns (idx, val, y)."""
    M, h = hidden.shape
    dev = hidden.device
    n = head.shape[0] if n_eff is None else int(n_eff)
    out_y = torch.empty((M, h), dtype=torch.bfloat16, device=dev) if out_y is None else out_y
    out_idx = torch.empty((M,), dtype=torch.int32, device=dev) if out_idx is None else out_idx
    out_val = torch.empty((M,), dtype=torch.float32, device=dev) if out_val is None else out_val
    L.mtp_draft_step(embed, embed.shape[0], token_ids, hidden, M, h, w_norm_embed, w_norm_hidden,
                     eps, norm_mode, fc, head, n, mask, mask_words, mask_stride_words, out_y,
                     out_idx, out_val, dev_err, stream)
    return out_idx, out_val, out_y


def paged_decode_attn(q, nkv, k_cache, v_cache, block_table, seq_len, k_scale=1.0, v_scale=1.0,
                      scale=None, out=None, ws=None, dev_err=None, stream=None):
    """Single-token decode attention of q [nq, hd] (bf16) over cache rows 0 .. seq_len - 1 of
    a paged E4M3 cache [num_blocks, block_size, nkv, hd]; returns (out, ws)."""
    nq, hd = q.shape
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    scale = 1.0 / float(hd) ** 0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty((nq, hd), dtype=torch.bfloat16, device=q.device)
    nbytes = L.mtp_paged_decode_attn_ws_bytes(nq, hd, seq_len)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    L.mtp_paged_decode_attn(q, nq, nkv, hd, k_cache, v_cache, block_table, block_table.numel(),
                            block_size, num_blocks, seq_len, k_scale, v_scale, scale, out, dev_err,
                            ws, ws.numel(), stream)
    return out, ws


def aligned_empty(nbytes: int, align: int, device) -> torch.Tensor:
    """A uint8 device buffer of nbytes whose address is a multiple of align (torch only
    promises 512 bytes)."""
    raw = torch.empty((nbytes + align,), dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % align
    return raw[off: off + nbytes]


def prefill_kv(inputs: dict, k_cache: torch.Tensor, v_cache: torch.Tensor, chunk_rows: int = 2048,
               ws: torch.Tensor | None = None, dev_err: torch.Tensor | None = None, stream=None):
    """Drafter-context prefill over device tensors named as in synth.prefill_inputs (plus the
    optional "norm_mode", "k_norm" [hd] and "in_norm" [h] entries)."""
    d = inputs
    R, h = d["hidden"].shape
    nkv, hd = int(d["nkv"]), int(d["hd"])
    chunk = min(int(chunk_rows), R)
    nbytes = L.mtp_prefill_ws_bytes(chunk, h, nkv, hd)
    if ws is None:
        ws = aligned_empty(nbytes, 1024, k_cache.device)
    L.mtp_prefill_kv(d["embed"], d["embed"].shape[0], d["tokens"], d["hidden"], R, h,
                     d["w_norm_embed"], d["w_norm_hidden"], d["eps"], int(d.get("norm_mode", 0)),
                     d["fc"], d["wk"], d["wv"], d.get("k_norm"), d.get("in_norm"), nkv, hd, d["rope_base"],
                     d["rope_pos"], int(d["cache_start"]),
                     d["block_table"], d["block_table"].numel(), int(d["block_size"]), k_cache,
                     v_cache, k_cache.shape[0], d["k_scale"], d["v_scale"], chunk, ws, ws.numel(),
                     dev_err, stream)
    return ws
