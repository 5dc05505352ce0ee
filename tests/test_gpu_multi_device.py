"""Calls on two devices in one process: kernel set-up (the dynamic
shared-memory size attribute, the occupancy query) belongs to each device's
context, so a quantiser and an fprop on cuda:0 and then on cuda:1 must both
work and both match the oracle (bit-exact codes; GEMM within the acceptance
bound). Skipped with fewer than two visible devices."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import assert_gemm_close, scale_bits, torch_bf16_to_np

pytestmark = pytest.mark.gpu


def _two_devices():
    import torch
    return torch.cuda.is_available() and torch.cuda.device_count() >= 2


@pytest.mark.skipif(not _two_devices(), reason="needs two CUDA devices")
def test_quantise_and_fprop_on_two_devices():
    import torch
    from blockwise_fp8_linear_fp8bw_b200 import ops
    m, n, k = 256, 384, 512
    x = S.bf16_normal((m, k), 0, 901, **S.X_DIST)
    w = S.bf16_normal((n, k), 0, 902, **S.W_DIST)
    rqx, rsx = oracle.quantize_rowwise(x)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False)
    acc, bound = oracle.gemm_fprop(rqx, rsx, rqw, rsw, with_bound=True)
    for d in (0, 1):
        dev = torch.device("cuda", d)
        tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        tw = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
        qx, sx = ops.quantize_rowwise(tx)
        qw, sw, _ = ops.quantize_weight_block(tw, transposed=False)
        y = ops.gemm_fprop(qx, sx, qw, sw)
        ops.fp8bw_check_device_error(device=dev)
        assert np.array_equal(qx.cpu().numpy(), rqx)
        assert np.array_equal(scale_bits(sx.cpu().numpy()), scale_bits(rsx))
        assert_gemm_close(torch_bf16_to_np(y), acc, bound, "fprop on %s" % dev)
