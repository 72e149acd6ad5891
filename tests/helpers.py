"""Test-side helpers: device transfers and the parity criteria.

Tolerances (floating point): |gpu - oracle| <= 2e-2 + 1e-2 * |oracle| per element,
the allclose reading of "abs <= 2e-2, rel <= 1e-2" against an fp64 oracle. Argmax:
exact wherever the oracle's top-2 (allowed) gap exceeds 1e-2, otherwise the GPU's
pick must be within 1e-2 of the oracle's maximum.
"""
import numpy as np
import torch

ATOL = 2e-2
RTOL = 1e-2
GAP = 1e-2


def to_dev_u16(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> a bf16 CUDA tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u16_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    err = np.abs(gpu - ref)
    lim = ATOL + RTOL * np.abs(ref)
    bad = np.nonzero(~(err <= lim))
    assert bad[0].size == 0, (f"{what}: {bad[0].size} elements out of tolerance; first at "
                              f"{tuple(b[0] for b in bad)} gpu={gpu[tuple(b[0] for b in bad)]} "
                              f"ref={ref[tuple(b[0] for b in bad)]} max_err={err.max()}")


def assert_argmax(idx_gpu: int, logits_ref: np.ndarray, allowed: np.ndarray | None = None):
    l = np.asarray(logits_ref, dtype=np.float64).copy()
    if allowed is not None:
        l[~allowed] = -np.inf
    order = np.argsort(-l, kind="stable")
    best = l[order[0]]
    second = l[order[1]] if l.size > 1 else -np.inf
    if best - second > GAP:
        assert idx_gpu == order[0], (idx_gpu, int(order[0]), best, second)
    else:
        assert allowed is None or allowed[idx_gpu]
        assert l[idx_gpu] >= best - GAP, (idx_gpu, l[idx_gpu], best)


def allowed_from_mask(mask_row: np.ndarray, n: int, mask_words: int) -> np.ndarray:
    words = np.asarray(mask_row, dtype=np.int32).view(np.uint32)[:mask_words]
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(-1)
    out = np.zeros(n, dtype=bool)
    m = min(n, bits.size)
    out[:m] = bits[:m]
    return out


def pad_scales(bscale: np.ndarray, k: int) -> np.ndarray:
    """[n, k/16] NVFP4 block scales -> the library's [n, pitch] layout (rows padded
    with zeros to a multiple of 16 bytes)."""
    n = bscale.shape[0]
    pitch = ((k // 16 + 15) // 16) * 16
    out = np.zeros((n, pitch), dtype=np.uint8)
    out[:, : k // 16] = bscale
    return out
