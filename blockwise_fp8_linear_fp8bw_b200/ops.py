"""Python binding of the C ABI: the same entry points, taking torch tensors.

Argument marshalling only (tensor -> device pointer, shape -> int64, the
current CUDA stream -> cudaStream_t); every step of the computation runs in
the CUDA library. The `fp8bw_*` functions take pre-allocated outputs; the
short-named helpers allocate the outputs with torch and call them.
"""
import ctypes

import torch

from . import _native

FP8BW_OK = 0
FP8BW_ERR_NULL = -1
FP8BW_ERR_SHAPE = -2
FP8BW_ERR_ALIGN = -3
FP8BW_ERR_DEVICE = -4
FP8BW_ERR_LAUNCH = -5
FP8BW_ERR_DEVICE_TIMEOUT = -6
FP8BW_ERR_CUDA = -7
FP8BW_ERR_ALIAS = -8
FP8BW_ERR_SCALE = -9

_lib = _native.load()


class Fp8bwError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        msg = _lib.fp8bw_status_string(status).decode()
        super().__init__("%s failed: %s (%d)" % (call, msg, status))


def _check(status: int, call: str) -> None:
    if status != FP8BW_OK:
        raise Fp8bwError(status, call)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream, dev=None):
    """The raw handle of `stream`; None means the current stream of `dev`
    (of the current device when `dev` is None). A torch stream must belong
    to `dev`."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    if hasattr(stream, "cuda_stream"):
        if dev is not None and stream.device != dev:
            raise ValueError("stream is on %s, the tensors on %s"
                             % (stream.device, dev))
        return stream.cuda_stream
    return int(stream)


def _device_of(tensors):
    """The one CUDA device that holds every (non-None) tensor."""
    devs = set()
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("expected a CUDA tensor")
        devs.add(t.device)
    if len(devs) != 1:
        raise ValueError("expected tensors on one CUDA device, got %s"
                         % sorted(str(d) for d in devs))
    return devs.pop()


def _call(name, tensors, stream, *args):
    """Call entry point `name` with `args` and the stream handle, on the
    device that holds `tensors`: the library launches on the current device,
    so a call for another device runs under a device guard."""
    dev = _device_of(tensors)
    handle = _stream(stream, dev)
    fn = getattr(_lib, name)
    if dev.index == torch.cuda.current_device():
        status = fn(*args, handle)
    else:
        with torch.cuda.device(dev):
            status = fn(*args, handle)
    _check(status, name)


def _expect(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected %s %s, got %s %s" %
                         (name, dtype, tuple(shape), t.dtype, tuple(t.shape)))


def _cdiv(a, b):
    return (a + b - 1) // b


def _fn(name, pow2):
    """The entry point, or its power-of-two-scale variant."""
    return name + "_pow2" if pow2 else name


# ----------------------------------------------------------- raw entry points

def fp8bw_quantize_rowwise(x, q, s, stream=None, pow2=False):
    rows, cols = x.shape
    _expect(x, torch.bfloat16, (rows, cols), "x")
    _expect(q, torch.uint8, (rows, cols), "q")
    _expect(s, torch.float32, (_cdiv(cols, 128), rows), "s")
    _call(_fn('fp8bw_quantize_rowwise', pow2), (x, q, s), stream,
          _ptr(x), rows, cols, _ptr(q), _ptr(s))


def fp8bw_quantize_colwise(x, q_t, s_t, q_row=None, s_row=None, stream=None,
                           pow2=False):
    rows, cols = x.shape
    _expect(x, torch.bfloat16, (rows, cols), "x")
    _expect(q_t, torch.uint8, (cols, rows), "q_t")
    _expect(s_t, torch.float32, (_cdiv(rows, 128), cols), "s_t")
    if q_row is not None:
        _expect(q_row, torch.uint8, (rows, cols), "q_row")
        _expect(s_row, torch.float32, (_cdiv(cols, 128), rows), "s_row")
    _call(_fn('fp8bw_quantize_colwise', pow2), (x, q_t, s_t, q_row, s_row),
          stream, _ptr(x), rows, cols, _ptr(q_t), _ptr(s_t), _ptr(q_row),
          _ptr(s_row))


def fp8bw_quantize_weight_block(w, q, s, q_t=None, stream=None,
                                pow2=False):
    n, k = w.shape
    _expect(w, torch.bfloat16, (n, k), "w")
    _expect(q, torch.uint8, (n, k), "q")
    _expect(s, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "s")
    if q_t is not None:
        _expect(q_t, torch.uint8, (k, n), "q_t")
    _call(_fn('fp8bw_quantize_weight_block', pow2), (w, q, s, q_t), stream,
          _ptr(w), n, k, _ptr(q), _ptr(s), _ptr(q_t))


def fp8bw_quantize_weight_block_batch(ws, qs, ss, q_ts=None, stream=None,
                                      pow2=False):
    """Block quantisation of up to 8 weights in one launch: job i is
    fp8bw_quantize_weight_block(ws[i], qs[i], ss[i], q_ts[i])."""
    count = len(ws)
    if q_ts is None:
        q_ts = [None] * count
    if not (len(qs) == len(ss) == len(q_ts) == count):
        raise ValueError("ws, qs, ss and q_ts must have one entry per weight")
    if count == 0:
        return
    jobs = (_native.WeightBlockJob * count)()
    tensors = []
    for i, (w, q, s, q_t) in enumerate(zip(ws, qs, ss, q_ts)):
        n, k = w.shape
        _expect(w, torch.bfloat16, (n, k), "ws[%d]" % i)
        _expect(q, torch.uint8, (n, k), "qs[%d]" % i)
        _expect(s, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "ss[%d]" % i)
        if q_t is not None:
            _expect(q_t, torch.uint8, (k, n), "q_ts[%d]" % i)
        jobs[i] = _native.WeightBlockJob(_ptr(w), n, k, _ptr(q), _ptr(s), _ptr(q_t))
        tensors += [w, q, s, q_t]
    _call(_fn("fp8bw_quantize_weight_block_batch", pow2), tensors, stream,
          ctypes.cast(jobs, ctypes.c_void_p), count)


def fp8bw_gemm_fprop(qx, sx, qw, sw, y, stream=None, pow2=False):
    m, k = qx.shape
    n = qw.shape[0]
    _expect(qx, torch.uint8, (m, k), "qx")
    _expect(qw, torch.uint8, (n, k), "qw")
    _expect(sx, torch.float32, (_cdiv(k, 128), m), "sx")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(y, torch.bfloat16, (m, n), "y")
    _call(_fn('fp8bw_gemm_fprop', pow2), (qx, sx, qw, sw, y), stream,
          _ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), m, n, k, _ptr(y))


def fp8bw_gemm_dgrad(qdy, sdy, qw, qw_is_transposed, sw, dx, stream=None,
                     pow2=False):
    m, n = qdy.shape
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    _expect(qdy, torch.uint8, (m, n), "qdy")
    _expect(qw, torch.uint8, (k, n) if qw_is_transposed else (n, k), "qw")
    _expect(sdy, torch.float32, (_cdiv(n, 128), m), "sdy")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(dx, torch.bfloat16, (m, k), "dx")
    _call(_fn('fp8bw_gemm_dgrad', pow2), (qdy, sdy, qw, sw, dx), stream,
          _ptr(qdy), _ptr(sdy), _ptr(qw), 1 if qw_is_transposed else 0,
          _ptr(sw), m, n, k, _ptr(dx))


def fp8bw_gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, dw, stream=None, pow2=False):
    n, m = qdy_t.shape
    k = qx_t.shape[0]
    _expect(qdy_t, torch.uint8, (n, m), "qdy_t")
    _expect(qx_t, torch.uint8, (k, m), "qx_t")
    _expect(sdy_t, torch.float32, (_cdiv(m, 128), n), "sdy_t")
    _expect(sx_t, torch.float32, (_cdiv(m, 128), k), "sx_t")
    _expect(dw, torch.bfloat16, (n, k), "dw")
    _call(_fn('fp8bw_gemm_wgrad', pow2), (qdy_t, sdy_t, qx_t, sx_t, dw),
          stream, _ptr(qdy_t), _ptr(sdy_t), _ptr(qx_t), _ptr(sx_t), m, n, k,
          _ptr(dw))


def fp8bw_gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, dw, accumulate=False,
                         stream=None, pow2=False):
    n, m = qdy_t.shape
    k = qx_t.shape[0]
    _expect(qdy_t, torch.uint8, (n, m), "qdy_t")
    _expect(qx_t, torch.uint8, (k, m), "qx_t")
    _expect(sdy_t, torch.float32, (_cdiv(m, 128), n), "sdy_t")
    _expect(sx_t, torch.float32, (_cdiv(m, 128), k), "sx_t")
    _expect(dw, torch.float32, (n, k), "dw")
    _call(_fn("fp8bw_gemm_wgrad_f32", pow2), (qdy_t, sdy_t, qx_t, sx_t, dw),
          stream, _ptr(qdy_t), _ptr(sdy_t), _ptr(qx_t), _ptr(sx_t), m, n, k,
          _ptr(dw), 1 if accumulate else 0)


def _wgrad_jobs(jobs, dtype):
    """ctypes array of fp8bw_wgrad_job from (qdy_t, sdy_t, qx_t, sx_t, dw)
    tuples, and the tensors it points into."""
    arr = (_native.WgradJob * len(jobs))()
    tensors = []
    for i, (qdy_t, sdy_t, qx_t, sx_t, dw) in enumerate(jobs):
        n, m = qdy_t.shape
        k = qx_t.shape[0]
        _expect(qdy_t, torch.uint8, (n, m), "jobs[%d].qdy_t" % i)
        _expect(qx_t, torch.uint8, (k, m), "jobs[%d].qx_t" % i)
        _expect(sdy_t, torch.float32, (_cdiv(m, 128), n), "jobs[%d].sdy_t" % i)
        _expect(sx_t, torch.float32, (_cdiv(m, 128), k), "jobs[%d].sx_t" % i)
        _expect(dw, dtype, (n, k), "jobs[%d].dw" % i)
        arr[i] = _native.WgradJob(_ptr(qdy_t), _ptr(sdy_t), _ptr(qx_t),
                                  _ptr(sx_t), m, n, k, _ptr(dw))
        tensors += [qdy_t, sdy_t, qx_t, sx_t, dw]
    return arr, tensors


def fp8bw_gemm_wgrad_batch(jobs, stream=None, pow2=False):
    """Up to 4 weight gradients over the same tokens in one launch: each job
    (qdy_t, sdy_t, qx_t, sx_t, dw) is fp8bw_gemm_wgrad of its arguments (bf16
    dw)."""
    if not jobs:
        return
    arr, tensors = _wgrad_jobs(jobs, torch.bfloat16)
    _call(_fn("fp8bw_gemm_wgrad_batch", pow2), tensors, stream,
          ctypes.cast(arr, ctypes.c_void_p), len(jobs))


def fp8bw_gemm_wgrad_f32_batch(jobs, accumulate=False, stream=None,
                               pow2=False):
    """The fp32-dW form of fp8bw_gemm_wgrad_batch (each job as
    fp8bw_gemm_wgrad_f32, the same `accumulate` for all)."""
    if not jobs:
        return
    arr, tensors = _wgrad_jobs(jobs, torch.float32)
    _call(_fn("fp8bw_gemm_wgrad_f32_batch", pow2), tensors, stream,
          ctypes.cast(arr, ctypes.c_void_p), len(jobs), 1 if accumulate else 0)


def fp8bw_gemm_fprop_quant(qx, sx, qw, sw, y, qy, sy, stream=None):
    m, k = qx.shape
    n = qw.shape[0]
    _expect(qx, torch.uint8, (m, k), "qx")
    _expect(qw, torch.uint8, (n, k), "qw")
    _expect(sx, torch.float32, (_cdiv(k, 128), m), "sx")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(y, torch.bfloat16, (m, n), "y")
    _expect(qy, torch.uint8, (m, n), "qy")
    _expect(sy, torch.float32, (_cdiv(n, 128), m), "sy")
    _call("fp8bw_gemm_fprop_quant", (qx, sx, qw, sw, y, qy, sy), stream,
          _ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), m, n, k, _ptr(y), _ptr(qy),
          _ptr(sy))


def fp8bw_gemm_dgrad_quant(qdy, sdy, qw, qw_is_transposed, sw, dx, qdx, sdx,
                           stream=None):
    m, n = qdy.shape
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    _expect(qdy, torch.uint8, (m, n), "qdy")
    _expect(qw, torch.uint8, (k, n) if qw_is_transposed else (n, k), "qw")
    _expect(sdy, torch.float32, (_cdiv(n, 128), m), "sdy")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(dx, torch.bfloat16, (m, k), "dx")
    _expect(qdx, torch.uint8, (m, k), "qdx")
    _expect(sdx, torch.float32, (_cdiv(k, 128), m), "sdx")
    _call("fp8bw_gemm_dgrad_quant", (qdy, sdy, qw, sw, dx, qdx, sdx), stream,
          _ptr(qdy), _ptr(sdy), _ptr(qw), 1 if qw_is_transposed else 0,
          _ptr(sw), m, n, k, _ptr(dx), _ptr(qdx), _ptr(sdx))


def fp8bw_gemm_fprop_quant_rowcol(qx, sx, qw, sw, y, qy, sy, qy_t, sy_t,
                                  stream=None):
    m, k = qx.shape
    n = qw.shape[0]
    _expect(qx, torch.uint8, (m, k), "qx")
    _expect(qw, torch.uint8, (n, k), "qw")
    _expect(sx, torch.float32, (_cdiv(k, 128), m), "sx")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(y, torch.bfloat16, (m, n), "y")
    _expect(qy, torch.uint8, (m, n), "qy")
    _expect(sy, torch.float32, (_cdiv(n, 128), m), "sy")
    _expect(qy_t, torch.uint8, (n, m), "qy_t")
    _expect(sy_t, torch.float32, (_cdiv(m, 128), n), "sy_t")
    _call("fp8bw_gemm_fprop_quant_rowcol", (qx, sx, qw, sw, y, qy, sy, qy_t, sy_t),
          stream, _ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), m, n, k, _ptr(y),
          _ptr(qy), _ptr(sy), _ptr(qy_t), _ptr(sy_t))


def fp8bw_gemm_dgrad_quant_rowcol(qdy, sdy, qw, qw_is_transposed, sw, dx, qdx,
                                  sdx, qdx_t, sdx_t, stream=None):
    m, n = qdy.shape
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    _expect(qdy, torch.uint8, (m, n), "qdy")
    _expect(qw, torch.uint8, (k, n) if qw_is_transposed else (n, k), "qw")
    _expect(sdy, torch.float32, (_cdiv(n, 128), m), "sdy")
    _expect(sw, torch.float32, (_cdiv(n, 128), _cdiv(k, 128)), "sw")
    _expect(dx, torch.bfloat16, (m, k), "dx")
    _expect(qdx, torch.uint8, (m, k), "qdx")
    _expect(sdx, torch.float32, (_cdiv(k, 128), m), "sdx")
    _expect(qdx_t, torch.uint8, (k, m), "qdx_t")
    _expect(sdx_t, torch.float32, (_cdiv(m, 128), k), "sdx_t")
    _call("fp8bw_gemm_dgrad_quant_rowcol",
          (qdy, sdy, qw, sw, dx, qdx, sdx, qdx_t, sdx_t), stream,
          _ptr(qdy), _ptr(sdy), _ptr(qw), 1 if qw_is_transposed else 0,
          _ptr(sw), m, n, k, _ptr(dx), _ptr(qdx), _ptr(sdx), _ptr(qdx_t),
          _ptr(sdx_t))


def _device_call(name, stream, device, *args):
    """Call a device-wide entry point (no tensor arguments) for one device:
    `device` if given, else the device of a torch `stream`, else the current
    device. The library works on the current device, so another device's
    call runs under a device guard."""
    if device is None and hasattr(stream, "device"):
        device = stream.device
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
        else torch.device(device)
    if dev.type != "cuda" or dev.index is None:
        raise ValueError("expected a CUDA device with an index, got %s" % dev)
    handle = _stream(stream, dev)
    fn = getattr(_lib, name)
    if dev.index == torch.cuda.current_device():
        status = fn(*args, handle)
    else:
        with torch.cuda.device(dev):
            status = fn(*args, handle)
    _check(status, name)


def fp8bw_selftest_wait_timeout(limit_ns, stream=None, device=None):
    _device_call("fp8bw_selftest_wait_timeout", stream, device, int(limit_ns))


def fp8bw_check_device_error(stream=None, device=None):
    """Synchronise `stream` and raise Fp8bwError if a kernel of the library on
    that device (`device`, else the stream's, else the current one) recorded
    an expired wait or a bad power-of-two scale since the last check."""
    _device_call("fp8bw_check_device_error", stream, device)


# ----------------------------------------------------------- allocating helpers

def quantize_rowwise(x, stream=None, pow2=False):
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    s = torch.empty((_cdiv(cols, 128), rows), dtype=torch.float32,
                    device=x.device)
    fp8bw_quantize_rowwise(x, q, s, stream, pow2=pow2)
    return q, s


def quantize_colwise(x, with_rowwise=False, stream=None, pow2=False):
    """-> (q_t, s_t) or (q_t, s_t, q_row, s_row) when with_rowwise."""
    rows, cols = x.shape
    dev = x.device
    q_t = torch.empty((cols, rows), dtype=torch.uint8, device=dev)
    s_t = torch.empty((_cdiv(rows, 128), cols), dtype=torch.float32,
                      device=dev)
    q_row = s_row = None
    if with_rowwise:
        q_row = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
        s_row = torch.empty((_cdiv(cols, 128), rows), dtype=torch.float32,
                            device=dev)
    fp8bw_quantize_colwise(x, q_t, s_t, q_row, s_row, stream, pow2=pow2)
    return (q_t, s_t, q_row, s_row) if with_rowwise else (q_t, s_t)


def quantize_weight_block(w, transposed=True, stream=None, pow2=False):
    n, k = w.shape
    dev = w.device
    q = torch.empty((n, k), dtype=torch.uint8, device=dev)
    s = torch.empty((_cdiv(n, 128), _cdiv(k, 128)), dtype=torch.float32,
                    device=dev)
    q_t = torch.empty((k, n), dtype=torch.uint8, device=dev) if transposed \
        else None
    fp8bw_quantize_weight_block(w, q, s, q_t, stream, pow2=pow2)
    return q, s, q_t


def gemm_fprop(qx, sx, qw, sw, stream=None, pow2=False):
    y = torch.empty((qx.shape[0], qw.shape[0]), dtype=torch.bfloat16,
                    device=qx.device)
    fp8bw_gemm_fprop(qx, sx, qw, sw, y, stream, pow2=pow2)
    return y


def gemm_dgrad(qdy, sdy, qw, sw, qw_is_transposed=True, stream=None,
               pow2=False):
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    dx = torch.empty((qdy.shape[0], k), dtype=torch.bfloat16,
                     device=qdy.device)
    fp8bw_gemm_dgrad(qdy, sdy, qw, qw_is_transposed, sw, dx, stream,
                     pow2=pow2)
    return dx


def gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, stream=None, pow2=False):
    dw = torch.empty((qdy_t.shape[0], qx_t.shape[0]), dtype=torch.bfloat16,
                     device=qdy_t.device)
    fp8bw_gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, dw, stream, pow2=pow2)
    return dw


def gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, main_grad=None, stream=None,
                   pow2=False):
    """fp32 dW; with `main_grad` given, dW is added into it in place and it is
    returned."""
    if main_grad is not None:
        fp8bw_gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, main_grad, True, stream,
                             pow2=pow2)
        return main_grad
    dw = torch.empty((qdy_t.shape[0], qx_t.shape[0]), dtype=torch.float32,
                     device=qdy_t.device)
    fp8bw_gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, dw, False, stream, pow2=pow2)
    return dw


def gemm_wgrad_batch(operands, stream=None, pow2=False):
    """-> [bf16 dW] for each (qdy_t, sdy_t, qx_t, sx_t) in `operands` (same
    token count), computed in one launch."""
    dws = [torch.empty((o[0].shape[0], o[2].shape[0]), dtype=torch.bfloat16,
                       device=o[0].device) for o in operands]
    fp8bw_gemm_wgrad_batch([tuple(o) + (dw,) for o, dw in zip(operands, dws)],
                           stream, pow2=pow2)
    return dws


def gemm_wgrad_f32_batch(operands, main_grads=None, stream=None, pow2=False):
    """fp32 dWs of fp8bw_gemm_wgrad_f32_batch; with `main_grads` given (one
    fp32 tensor per job), each dW is added into its main-grad in place and the
    main-grads are returned."""
    if main_grads is not None:
        fp8bw_gemm_wgrad_f32_batch([tuple(o) + (g,) for o, g in zip(operands, main_grads)],
                                   True, stream, pow2=pow2)
        return list(main_grads)
    dws = [torch.empty((o[0].shape[0], o[2].shape[0]), dtype=torch.float32,
                       device=o[0].device) for o in operands]
    fp8bw_gemm_wgrad_f32_batch([tuple(o) + (dw,) for o, dw in zip(operands, dws)],
                               False, stream, pow2=pow2)
    return dws


def gemm_fprop_quant(qx, sx, qw, sw, stream=None):
    """-> (y, qy, sy): the bf16 product and its row-wise quantisation."""
    m, n = qx.shape[0], qw.shape[0]
    dev = qx.device
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    qy = torch.empty((m, n), dtype=torch.uint8, device=dev)
    sy = torch.empty((_cdiv(n, 128), m), dtype=torch.float32, device=dev)
    fp8bw_gemm_fprop_quant(qx, sx, qw, sw, y, qy, sy, stream)
    return y, qy, sy


def gemm_dgrad_quant(qdy, sdy, qw, sw, qw_is_transposed=True, stream=None):
    """-> (dx, qdx, sdx): the bf16 product and its row-wise quantisation."""
    m = qdy.shape[0]
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    dev = qdy.device
    dx = torch.empty((m, k), dtype=torch.bfloat16, device=dev)
    qdx = torch.empty((m, k), dtype=torch.uint8, device=dev)
    sdx = torch.empty((_cdiv(k, 128), m), dtype=torch.float32, device=dev)
    fp8bw_gemm_dgrad_quant(qdy, sdy, qw, qw_is_transposed, sw, dx, qdx, sdx,
                           stream)
    return dx, qdx, sdx


def gemm_fprop_quant_rowcol(qx, sx, qw, sw, stream=None):
    """-> (y, qy, sy, qy_t, sy_t): the bf16 product with its row-wise and its
    transposed column-wise quantisation."""
    m, n = qx.shape[0], qw.shape[0]
    dev = qx.device
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    qy = torch.empty((m, n), dtype=torch.uint8, device=dev)
    sy = torch.empty((_cdiv(n, 128), m), dtype=torch.float32, device=dev)
    qy_t = torch.empty((n, m), dtype=torch.uint8, device=dev)
    sy_t = torch.empty((_cdiv(m, 128), n), dtype=torch.float32, device=dev)
    fp8bw_gemm_fprop_quant_rowcol(qx, sx, qw, sw, y, qy, sy, qy_t, sy_t, stream)
    return y, qy, sy, qy_t, sy_t


def gemm_dgrad_quant_rowcol(qdy, sdy, qw, sw, qw_is_transposed=True,
                            stream=None):
    """-> (dx, qdx, sdx, qdx_t, sdx_t): the bf16 product with its row-wise
    and its transposed column-wise quantisation."""
    m = qdy.shape[0]
    k = qw.shape[0] if qw_is_transposed else qw.shape[1]
    dev = qdy.device
    dx = torch.empty((m, k), dtype=torch.bfloat16, device=dev)
    qdx = torch.empty((m, k), dtype=torch.uint8, device=dev)
    sdx = torch.empty((_cdiv(k, 128), m), dtype=torch.float32, device=dev)
    qdx_t = torch.empty((k, m), dtype=torch.uint8, device=dev)
    sdx_t = torch.empty((_cdiv(m, 128), k), dtype=torch.float32, device=dev)
    fp8bw_gemm_dgrad_quant_rowcol(qdy, sdy, qw, qw_is_transposed, sw, dx, qdx,
                                  sdx, qdx_t, sdx_t, stream)
    return dx, qdx, sdx, qdx_t, sdx_t


def quantize_weight_block_batch(ws, transposed=True, stream=None, pow2=False):
    """-> [(q, s, q_t)] for each weight, all quantised in one launch."""
    out = []
    for w in ws:
        n, k = w.shape
        dev = w.device
        out.append((torch.empty((n, k), dtype=torch.uint8, device=dev),
                    torch.empty((_cdiv(n, 128), _cdiv(k, 128)), dtype=torch.float32,
                                device=dev),
                    torch.empty((k, n), dtype=torch.uint8, device=dev)
                    if transposed else None))
    fp8bw_quantize_weight_block_batch(ws, [o[0] for o in out], [o[1] for o in out],
                                      [o[2] for o in out], stream, pow2=pow2)
    return out
