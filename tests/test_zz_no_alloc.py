"""fp8blk_linear_w8a8_noalloc: the W8A8 linear for callers that cannot give
the library a workspace (a runtime that forbids device allocations once it
is serving, or code that must not call cudaMalloc because it can synchronize
the device). It borrows a fixed scratch array built into the library instead.

These tests call it through the C ABI, two calls in a row -- the second one
smaller than the first, so it runs over the scratch the first call left
behind. Each output must equal the workspace-taking fp8blk_linear_w8a8's on
the same inputs bit for bit (the same kernels on the same codes, only the
scratch differs), and lie within the linear tolerance of the CPU oracle's
W8A8 result. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import block_scaled_fp8_fp8blk_b200 as fb
import oracle
from block_scaled_fp8_fp8blk_b200 import synth, workloads as W
from helpers import bf16_to_f64, check_linear

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCRATCH_BYTES = 16 * 1024 * 1024   # FP8BLK_NOALLOC_SCRATCH_BYTES in include/fp8blk.h


def padded_bf16(t, ld):
    R, C = t.shape
    buf = torch.zeros((R, ld), dtype=torch.bfloat16, device=DEV)
    buf[:, :C] = t.to(DEV)
    return buf[:, :C]


def noalloc(x, q, s, y):
    M, K = x.shape
    N = q.shape[0]
    return fb.lib().fp8blk_linear_w8a8_noalloc(
        x.data_ptr(), x.stride(0), q.data_ptr(), q.stride(0), s.data_ptr(), y.data_ptr(),
        y.stride(0), M, N, K, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_w8a8_and_the_oracle_on_two_calls_in_a_row():
    torch.cuda.set_device(0)
    cases = [W.Workload("first_m1024_k5120_n2048", 1024, 5120, 2048),
             W.Workload("second_m77_k1000_n1000", 77, 1000, 1000, row_gain_sigma=0.5)]
    for wl in cases:
        assert fb.workspace_size(1, wl.M, wl.N, wl.K) <= SCRATCH_BYTES
        w, xh = wl.weight_bf16(), wl.x_bf16()
        x = padded_bf16(xh, -(-wl.K // 8) * 8)
        q, s = fb.quantize_weight(w.to(DEV))
        ref = fb.linear_w8a8(x, q, s)
        y = torch.full((wl.M, -(-wl.N // 8) * 8), float("nan"), dtype=torch.bfloat16,
                       device=DEV)[:, :wl.N]
        assert noalloc(x, q, s, y) == 0
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), wl.name
        rows = wl.checked_rows(64)
        qx, sx = oracle.act_quant(synth.bf16_bits(xh))
        want = oracle.linear_w8a8(qx, sx, q.cpu().numpy(), s.cpu().numpy(), wl.N, wl.K, rows=rows)
        check_linear(bf16_to_f64(y)[rows], want, f"noalloc/{wl.name}")
    assert fb.read_device_error() == 0


def test_noalloc_refuses_problems_larger_than_its_scratch():
    torch.cuda.set_device(0)
    M, K, N = 4096, 5120, 256
    assert fb.workspace_size(1, M, N, K) > SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((N, K), dtype=torch.uint8, device=DEV)
    s = torch.zeros((N // 128, K // 128), dtype=torch.float32, device=DEV)
    y = torch.zeros((M, N), dtype=torch.bfloat16, device=DEV)
    assert noalloc(x, q, s, y) == 4   # FP8BLK_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0
