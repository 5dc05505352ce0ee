"""Host logic of the Python binding without a GPU: which device and stream a
call goes to, and which arguments it refuses before reaching the library.
The library is replaced by a recorder and the tensors by stand-ins that carry
a CUDA device, so nothing is launched."""
import contextlib

import pytest
import torch

from blockwise_fp8_linear_fp8bw_b200 import ops


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("fp8bw_"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append((name, args, _State.device))
            return 0
        return call


class _State:
    current = 0        # torch's current CUDA device
    device = 0         # the device the library would launch on


class _Tensor:
    """Stand-in for a contiguous CUDA tensor."""
    _next = [0x10000]

    def __init__(self, shape, dtype, device=0, cuda=True):
        self.shape, self.dtype, self.is_cuda = tuple(shape), dtype, cuda
        self.device = torch.device("cuda", device) if cuda else torch.device("cpu")
        _Tensor._next[0] += 0x1000
        self._ptr = _Tensor._next[0]

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return self._ptr


class _Stream:
    def __init__(self, device, handle):
        self.device, self.cuda_stream = torch.device("cuda", device), handle


@pytest.fixture
def lib(monkeypatch):
    rec = _Recorder()
    _State.current = _State.device = 0

    @contextlib.contextmanager
    def guard(dev):
        prev = _State.device
        _State.device = torch.device(dev).index
        try:
            yield
        finally:
            _State.device = prev

    monkeypatch.setattr(ops, "_lib", rec)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: _State.current)
    monkeypatch.setattr(torch.cuda, "device", guard)
    monkeypatch.setattr(
        torch.cuda, "current_stream",
        lambda device=None: _Stream(_State.current if device is None
                                    else torch.device(device).index,
                                    1000 + (_State.current if device is None
                                            else torch.device(device).index)))
    return rec


def _fprop_args(dev=0, m=256, n=384, k=512):
    u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
    return (_Tensor((m, k), u8, dev), _Tensor((k // 128, m), f32, dev),
            _Tensor((n, k), u8, dev), _Tensor((n // 128, k // 128), f32, dev),
            _Tensor((m, n), bf, dev))


def test_current_device_call_passes_pointers_sizes_and_stream(lib):
    qx, sx, qw, sw, y = _fprop_args()
    ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y)
    name, args, dev = lib.calls[-1]
    assert name == "fp8bw_gemm_fprop" and dev == 0
    assert args == (qx.data_ptr(), sx.data_ptr(), qw.data_ptr(), sw.data_ptr(),
                    256, 384, 512, y.data_ptr(), 1000)


def test_tensors_on_another_device_run_under_its_guard(lib):
    # torch's current device is 0; the tensors live on device 1: the library
    # must see device 1 current and get device 1's current stream.
    qx, sx, qw, sw, y = _fprop_args(dev=1)
    ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y, pow2=True)
    name, args, dev = lib.calls[-1]
    assert name == "fp8bw_gemm_fprop_pow2" and dev == 1 and args[-1] == 1001
    assert _State.device == 0          # guard restored


def test_mixed_devices_are_refused_before_the_library(lib):
    qx, sx, qw, sw, _ = _fprop_args(dev=0)
    y = _Tensor((256, 384), torch.bfloat16, device=1)
    with pytest.raises(ValueError, match="one CUDA device"):
        ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y)
    assert lib.calls == []


def test_stream_of_another_device_is_refused(lib):
    qx, sx, qw, sw, y = _fprop_args(dev=0)
    with pytest.raises(ValueError, match="stream"):
        ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y, stream=_Stream(1, 55))
    assert lib.calls == []
    ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y, stream=_Stream(0, 55))
    assert lib.calls[-1][1][-1] == 55
    ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y, stream=77)      # raw handle
    assert lib.calls[-1][1][-1] == 77


def test_cpu_tensor_and_wrong_code_dtype_are_refused(lib):
    qx, sx, qw, sw, y = _fprop_args()
    cpu_y = _Tensor((256, 384), torch.bfloat16, cuda=False)
    with pytest.raises(ValueError, match="CUDA"):
        ops.fp8bw_gemm_fprop(qx, sx, qw, sw, cpu_y)
    bad_qx = _Tensor((256, 512), torch.bfloat16)
    with pytest.raises(ValueError, match="qx"):
        ops.fp8bw_gemm_fprop(bad_qx, sx, qw, sw, y)
    bad_qdy_t = _Tensor((384, 256), torch.float32)
    with pytest.raises(ValueError, match="qdy_t"):
        ops.fp8bw_gemm_wgrad(bad_qdy_t, _Tensor((2, 384), torch.float32),
                             _Tensor((512, 256), torch.uint8),
                             _Tensor((2, 512), torch.float32),
                             _Tensor((384, 512), torch.bfloat16))
    assert lib.calls == []


def test_optional_outputs_may_be_absent(lib):
    x = _Tensor((256, 512), torch.bfloat16, device=1)
    q_t = _Tensor((512, 256), torch.uint8, device=1)
    s_t = _Tensor((2, 512), torch.float32, device=1)
    ops.fp8bw_quantize_colwise(x, q_t, s_t)
    name, args, dev = lib.calls[-1]
    assert name == "fp8bw_quantize_colwise" and dev == 1
    assert args == (x.data_ptr(), 256, 512, q_t.data_ptr(), s_t.data_ptr(),
                    None, None, 1001)


def test_device_error_check_goes_to_the_stream_or_given_device(lib):
    # the error record is per device: a check for device 1 must run with
    # device 1 current and device 1's stream, whatever torch's current one is
    ops.fp8bw_check_device_error(_Stream(1, 66))
    name, args, dev = lib.calls[-1]
    assert name == "fp8bw_check_device_error" and dev == 1 and args == (66,)
    ops.fp8bw_check_device_error(device=1)
    assert lib.calls[-1] == ("fp8bw_check_device_error", (1001,), 1)
    ops.fp8bw_check_device_error()
    assert lib.calls[-1] == ("fp8bw_check_device_error", (1000,), 0)
    with pytest.raises(ValueError, match="stream"):
        ops.fp8bw_check_device_error(_Stream(0, 5), device=1)
    ops.fp8bw_selftest_wait_timeout(1000, device=1)
    assert lib.calls[-1] == ("fp8bw_selftest_wait_timeout", (1000, 1001), 1)
    assert _State.device == 0


def test_data_parallel_default_stream_is_the_shards_device(lib, monkeypatch):
    from blockwise_fp8_linear_fp8bw_b200 import data_parallel as dp
    n, k, m = 256, 384, 512
    u8, f32 = torch.uint8, torch.float32
    qdy_t, sdy_t = _Tensor((n, m), u8, 1), _Tensor((m // 128, n), f32, 1)
    qx_t, sx_t = _Tensor((k, m), u8, 1), _Tensor((m // 128, k), f32, 1)
    made = []

    def fake_empty(shape, dtype, device):
        t = _Tensor(shape, dtype, torch.device(device).index)
        made.append(t)
        return t
    monkeypatch.setattr(torch, "empty", fake_empty)
    monkeypatch.setattr(torch.distributed, "is_initialized", lambda: False)
    dw = dp.wgrad_all_reduce(qdy_t, sdy_t, qx_t, sx_t)
    name, args, dev = lib.calls[-1]
    assert name == "fp8bw_gemm_wgrad_f32" and dev == 1
    assert args[-1] == 1001 and dw is made[-1]
