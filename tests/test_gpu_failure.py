"""Failure detection without a GPU fault: a device-side wait on a barrier that nothing
completes runs out after a short limit, records FPX_ERR_TIMEOUT, and the context stays usable
(the next prefill on the same stream is correct)."""
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx
from gen import WORKLOADS, generate
import parity as PT

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    lib = fpx.load()
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.fpx_diag_bounded_wait(ws.data_ptr(), 20_000_000, stream) == 0  # 20 ms
    assert fpx.status(ws) == -6  # FPX_ERR_TIMEOUT recorded, kernel returned
    fpx.clear_status(ws)
    assert fpx.status(ws) == 0
    # the context is still usable: a full prefill on the same stream is correct
    w = WORKLOADS["llama8b_bf16_n8192"].with_(seqlens=(700,), hq=2, hkv=1)
    dev = PT.to_device(generate(w))
    out = fpx.prefill(dev["q"], dev["k"], dev["v"], w.block, 0.0, dev["cu_seqlens"])
    q = dev["q"].transpose(0, 1)[None].float()
    k = dev["k"].transpose(0, 1)[None].float().repeat_interleave(2, 1)
    v = dev["v"].transpose(0, 1)[None].float().repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0].transpose(0, 1)
    assert (out["o"].float() - ref).abs().max().item() < 2e-2


def test_bounded_wait_argument_checks():
    lib = fpx.load()
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert lib.fpx_diag_bounded_wait(None, 1000, None) == -1
    assert lib.fpx_diag_bounded_wait(ws.data_ptr(), 0, None) == -1
    assert lib.fpx_diag_bounded_wait(ws.data_ptr(), 3_000_000_000, None) == -1
    assert lib.fpx_diag_bounded_wait(ws.data_ptr() + 16, 1000, None) == -3
