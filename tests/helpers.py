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
