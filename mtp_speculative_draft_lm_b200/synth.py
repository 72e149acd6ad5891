"""Seeded synthetic inputs for the draft-head hot path.

This module only draws and lays out input data (torch's CPU generator, so the same
seed gives the same bytes on any machine with this torch build). It holds none of
the method's arithmetic and is the one module that both the CPU oracle's tests and
the CUDA path's tests and benchmark read their inputs from.

Workloads (shapes from the draft-head pages: the 154,880 x 4,096 BF16 draft head of
metrale_model_arch/glm5next_mtp_head/init.rs, the 32k-token / hidden-5120 prompt
buffer sizing of spark_model/layers/mtp_head.rs, block size 16):

* ``tiny_draft``   hidden 256, vocab 4096: embedding and lm_head tables, fc, norms.
* ``head_table``   a [N, K] bf16 table ~N(0, 0.02) with, per input row m, two planted
  rows: ``top[m]`` = bf16(a * x_m) whose logit is about ``t_top`` and ``second[m]``
  with logit about ``t_second``, far above the ~N(0, 1.3^2) random logits. A mask
  (optional) keeps a seeded fraction of tokens, always keeps ``second[m]`` and always
  drops ``top[m]``, so a masked argmax must skip the larger decoy.
* ``prefill_inputs`` prompt rows, token ids, tables and a seeded block-table
  permutation for the drafter-context prefill.
"""
from __future__ import annotations

import numpy as np
import torch

TINY = dict(seed=1001, vocab=4096, h=256)
BF16_HEAD = dict(seed=1002, N=154880, K=4096, Ms=(1, 2, 4))
FP8_HEAD = dict(seed=1003, N=154880, K=4096, Ms=(1, 4, 8), mask_keep=0.1)
NVFP4_HEAD = dict(seed=1004, N=131072, K=5120, Ms=(1, 4, 16))
PREFILL = dict(seed=1005, R=32768, vocab=131072, h=5120, nkv=8, hd=128, chunk=2048,
               rope_base=1e6, block_size=16, eps=1e-6)

_CHUNK_ROWS = 8192


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(g: torch.Generator, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """bf16 tensor of N(mean, std^2) draws, generated in row chunks (bounded memory)."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(shape[0], -1) if len(shape) > 1 else out.view(-1, 1)
    for r0 in range(0, flat.shape[0], _CHUNK_ROWS):
        r1 = min(flat.shape[0], r0 + _CHUNK_ROWS)
        t = torch.randn((r1 - r0, flat.shape[1]), generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        if mean != 0.0:
            t.add_(mean)
        flat[r0:r1].copy_(t)
    return out


def as_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (no copy when contiguous)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def pack_mask(allowed: np.ndarray) -> np.ndarray:
    """[M, N] bool -> [M, ceil(N/32)] int32 words; token t is bit t%32 of word t//32."""
    allowed = np.asarray(allowed, dtype=bool)
    M, N = allowed.shape
    words = (N + 31) // 32
    bits = np.zeros((M, words * 32), dtype=np.uint64)
    bits[:, :N] = allowed
    w = (bits.reshape(M, words, 32) << np.arange(32, dtype=np.uint64)).sum(axis=2)
    return w.astype(np.uint32).view(np.int32)


def keep_mask(seed: int, M: int, N: int, keep: float) -> tuple[np.ndarray, np.ndarray]:
    """Per-row grammar masks keeping a seeded fraction `keep` of N tokens: ([M, N] bool
    allowed, [M, ceil(N/32)] int32 packed words)."""
    g = _gen(seed)
    allowed = (torch.rand((M, N), generator=g) < keep).numpy()
    return allowed, pack_mask(allowed)


def tiny_draft(seed: int = TINY["seed"], vocab: int = TINY["vocab"], h: int = TINY["h"],
               M: int = 1) -> dict:
    g = _gen(seed)
    embed = normal_bf16(g, (vocab, h), 0.02)
    lm_head = normal_bf16(g, (vocab, h), 0.02)
    fc = normal_bf16(g, (h, 2 * h), 0.02)
    w_ne = normal_bf16(g, (h,), 0.01, 1.0)
    w_nh = normal_bf16(g, (h,), 0.01, 1.0)
    hidden = normal_bf16(g, (M, h), 1.0)
    tokens = torch.randint(0, vocab, (M,), generator=g, dtype=torch.int32)
    return dict(embed=embed, lm_head=lm_head, fc=fc, w_norm_embed=w_ne, w_norm_hidden=w_nh,
                hidden=hidden, tokens=tokens, eps=1e-6, vocab=vocab, h=h)


def head_table(seed: int, N: int, K: int, M: int, t_top: float = 14.0,
               t_second: float = 10.0, mask_keep: float | None = None,
               std: float = 0.02) -> dict:
    """[N, K] bf16 table with planted rows; inputs x [M, K] ~ N(0, 1)."""
    g = _gen(seed)
    W = normal_bf16(g, (N, K), std)
    x = normal_bf16(g, (M, K), 1.0)
    picks = torch.randperm(N, generator=g)[: 2 * M]
    top = picks[:M].to(torch.int64)
    second = picks[M: 2 * M].to(torch.int64)
    xf = x.to(torch.float64)
    n2 = (xf * xf).sum(dim=1)
    for m in range(M):
        W[int(top[m])] = (xf[m] * (t_top / n2[m])).to(torch.bfloat16)
        W[int(second[m])] = (xf[m] * (t_second / n2[m])).to(torch.bfloat16)
    out = dict(W=W, x=x, top=top.numpy(), second=second.numpy(), N=N, K=K, M=M)
    if mask_keep is not None:
        allowed = (torch.rand((M, N), generator=g) < mask_keep).numpy()
        for m in range(M):
            allowed[m, int(top[m])] = False
            allowed[m, int(second[m])] = True
        out["mask"] = pack_mask(allowed)
        out["allowed"] = allowed
    return out


def prefill_inputs(seed: int = PREFILL["seed"], R: int = PREFILL["R"],
                   vocab: int = PREFILL["vocab"], h: int = PREFILL["h"],
                   nkv: int = PREFILL["nkv"], hd: int = PREFILL["hd"],
                   block_size: int = PREFILL["block_size"], extra_blocks: int = 1) -> dict:
    g = _gen(seed)
    tokens = torch.randint(0, vocab, (R,), generator=g, dtype=torch.int32)
    embed = normal_bf16(g, (vocab, h), 0.02)
    hidden = normal_bf16(g, (R, h), 1.0)
    fc = normal_bf16(g, (h, 2 * h), 0.02)
    wk = normal_bf16(g, (nkv * hd, h), 0.02)
    wv = normal_bf16(g, (nkv * hd, h), 0.02)
    w_ne = normal_bf16(g, (h,), 0.01, 1.0)
    w_nh = normal_bf16(g, (h,), 0.01, 1.0)
    num_blocks = R // block_size + extra_blocks
    block_table = torch.randperm(num_blocks, generator=g).to(torch.int32)
    rope_pos = torch.arange(1, R + 1, dtype=torch.int32)
    return dict(tokens=tokens, embed=embed, hidden=hidden, fc=fc, wk=wk, wv=wv,
                w_norm_embed=w_ne, w_norm_hidden=w_nh, block_table=block_table,
                num_blocks=num_blocks, rope_pos=rope_pos, cache_start=0, R=R, vocab=vocab,
                h=h, nkv=nkv, hd=hd, block_size=block_size, eps=PREFILL["eps"],
                rope_base=PREFILL["rope_base"], k_scale=1.0, v_scale=1.0)
