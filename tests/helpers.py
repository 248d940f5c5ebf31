"""Shared test helpers: oracle-side references for a workload and the
tolerance check of the linear layer."""
from __future__ import annotations

import numpy as np

import oracle
from block_scaled_fp8_fp8blk_b200 import synth

# Tolerances of the linear layer against the FP64 oracle of the same mode:
# relative Frobenius error and a per-element bound.
REL_FRO = 2e-3
ELEM_REL = 2.0 ** -7
ELEM_RMS = 1e-2


def bf16_bits(t) -> np.ndarray:
    """torch bfloat16 tensor (any device) -> numpy uint16 bit patterns."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t) -> np.ndarray:
    b = bf16_bits(t)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_linear(y: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    """y (float64 image of the BF16 output) against the FP64 oracle."""
    assert y.shape == ref.shape, (y.shape, ref.shape)
    err = y - ref
    nref = np.linalg.norm(ref)
    rel = float(np.linalg.norm(err) / nref) if nref > 0 else float(np.linalg.norm(err))
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    bound = ELEM_REL * np.abs(ref) + ELEM_RMS * rms
    worst = float(np.max(np.abs(err) - bound)) if ref.size else -1.0
    stats = {"rel_fro": rel, "rms": rms, "worst_excess": worst}
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert worst <= 0, f"{what}: per-element bound exceeded by {worst:.3e} ({stats})"
    return stats


def weight_bits(wl) -> np.ndarray:
    return synth.bf16_bits(wl.weight_bf16())


def x_bits(wl) -> np.ndarray:
    return synth.bf16_bits(wl.x_bf16())


def oracle_refs(wl, wb: np.ndarray, xb: np.ndarray, rows=None):
    """(q, s, ref_w8a16[rows], ref_w8a8[rows], qx, sx) from the oracle alone."""
    q, s = oracle.quantize_weight(wb)
    qx, sx = oracle.act_quant(xb)
    r16 = oracle.linear_w8a16(xb, q, s, wl.N, wl.K, rows=rows)
    r8 = oracle.linear_w8a8(qx, sx, q, s, wl.N, wl.K, rows=rows)
    return q, s, r16, r8, qx, sx


def e4m3_midpoints(limit: float) -> np.ndarray:
    """Every positive value halfway between two neighbouring E4M3 values, up to limit."""
    sub = (2 * np.arange(7) + 1) * 2.0 ** -10
    norm = [(1 + (2 * j + 1) / 16) * 2.0 ** e for e in range(-6, 9) for j in range(8)]
    m = np.concatenate([sub, np.array(norm)])
    return m[m <= limit]


def tie_heavy_weight() -> np.ndarray:
    """BF16 bits of a 200 x 300 weight whose quotients v / s sit exactly on
    E4M3 decision points in controlled numbers. Block (0, 0) has amax 448
    (s = 1) and per warp of 16 rows 0, 5, 31, 33, 40, 63, 64 or 65 ties.
    Block (0, 1) is all ties at amax 896 (s = 2). Ties also sit on the last
    columns of block (0, 2), which is 44 columns wide, and on the last rows
    of block (1, 0), which is 72 rows high. Block (1, 2) is all ties. All
    other values have 8 significant bits, so they are never a tie at
    s = 1 or 2."""
    rng = np.random.default_rng(77)
    N, K = 200, 300
    mids = e4m3_midpoints(432.0)
    base = synth.bf16_bits(synth.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 60.0))
    base = base | np.uint16(1)
    w = (base.astype(np.uint32) << 16).view(np.float32).copy()
    np.clip(w, -440.0, 440.0, out=w)
    w = synth.bf16_bits(synth.to_bf16(w)) | np.uint16(1)
    w = (w.astype(np.uint32) << 16).view(np.float32).copy()

    def ties(n):
        return rng.choice(mids, n) * rng.choice([-1.0, 1.0], n)

    for wi, n in enumerate([0, 5, 31, 33, 40, 63, 64, 65]):
        pos = rng.choice(16 * 128, n, replace=False)
        w[16 * wi + pos // 128, pos % 128] = ties(n)
    w[0, 0] = 448.0
    w[:128, 128:256] = 2.0 * ties(128 * 128).reshape(128, 128)
    w[77, 200] = -896.0
    w[:128, 290:300] = ties(1280).reshape(128, 10)
    w[3, 256] = 448.0
    w[190:200, :128] = ties(1280).reshape(10, 128)
    w[128, 5] = 448.0
    w[128:200, 256:300] = ties(72 * 44).reshape(72, 44)
    w[199, 299] = 448.0
    wb = synth.bf16_bits(synth.to_bf16(w))
    assert np.array_equal((wb.astype(np.uint32) << 16).view(np.float32), w), "values must be BF16"
    return wb
