"""The error path of the bounded device-side waits, on the GPU without a
fault: a wait on a barrier that nothing completes gives up after its limit,
the host reads FP8BW_ERR_DEVICE_TIMEOUT, the record is cleared, and the
context keeps working (a GEMM afterwards is correct)."""
import pytest

import oracle
import synthetic as S
from helpers import assert_gemm_close, bf16_np_to_torch, torch_bf16_to_np

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    import time
    from blockwise_fp8_linear_fp8bw_b200 import ops
    ops.fp8bw_check_device_error()                 # start clean
    t0 = time.perf_counter()
    ops.fp8bw_selftest_wait_timeout(20_000_000)    # 20 ms
    with pytest.raises(ops.Fp8bwError) as e:
        ops.fp8bw_check_device_error()
    assert e.value.status == ops.FP8BW_ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 >= 0.02        # it did wait
    ops.fp8bw_check_device_error()                 # cleared
    # the context is still usable
    x = S.bf16_normal((256, 256), 0, 901, **S.X_DIST)
    w = S.bf16_normal((256, 256), 0, 902, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x))
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w), transposed=False)
    y = torch_bf16_to_np(ops.gemm_fprop(qx, sx, qw, sw))
    ops.fp8bw_check_device_error()
    rqx, rsx = oracle.quantize_rowwise(x)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False)
    acc, bound = oracle.gemm_fprop(rqx, rsx, rqw, rsw, with_bound=True)
    assert_gemm_close(y, acc, bound, "fprop after an expired wait")
