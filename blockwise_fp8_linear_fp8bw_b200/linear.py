"""A training linear layer on the library's blockwise-FP8 path.

Y = X W^T with the E4M3 quantisers and GEMMs of this library (Puro-2B report:
arxiv-wiki summary, "Approach" item (4) -- E4M3, 1x128 activation groups,
128x128 weight blocks; paperlayer.ai summary, Appendix C, "FP8 implementation
pipeline" -- forward, data-gradient and weight-gradient GEMMs in E4M3, bf16
hidden flow, fp32 gradients):

  forward   W -> 128x128 block codes (+ transposed codes for dgrad)
            X -> row-wise (fprop) and column-wise (wgrad) codes, one pass
            Y = fprop(X, W)                                        bf16
  backward  dY -> row-wise (dgrad) and column-wise (wgrad) codes, one pass
            dX = dgrad(dY, W)                                      bf16
            dW = wgrad(dY, X): added in fp32 into weight.main_grad when the
                 weight carries one (gradient accumulation over
                 micro-batches; the add is done by the GEMM's epilogue, for
                 either scale form), else returned in the weight's dtype.

Linears that feed one another directly (BlockwiseFp8Chain) fuse the
quantisation of every intermediate activation and gradient into the GEMM that
produces it (row-wise and column-wise codes from the fprop / dgrad epilogue).

Every step runs in the CUDA library; this module only reshapes tensors and
keeps the codes the backward pass needs. Inputs must be bf16 CUDA tensors
whose dimensions are multiples of 16.
"""
import torch

from . import ops

_WEIGHT_BATCH = 8     # weights per batched block-quantisation launch
_WGRAD_BATCH = 4      # weight gradients per batched wgrad launch


def _rows(t, k):
    if not t.is_cuda or t.dtype != torch.bfloat16:
        raise ValueError("expected a bf16 CUDA tensor, got %s on %s"
                         % (t.dtype, t.device))
    return t.reshape(-1, k).contiguous()


class BlockwiseFp8LinearFunction(torch.autograd.Function):
    """y = x @ weight.T on the blockwise-FP8 path (see the module docstring).
    `pow2` selects the power-of-two-scale variant."""

    @staticmethod
    def forward(ctx, x, weight, pow2=False):
        n, k = weight.shape
        x2 = _rows(x, k)
        w = _rows(weight, k)
        qw, sw, qw_t = ops.quantize_weight_block(w, transposed=True, pow2=pow2)
        qx_t, sx_t, qx, sx = ops.quantize_colwise(x2, with_rowwise=True,
                                                  pow2=pow2)
        y = ops.gemm_fprop(qx, sx, qw, sw, pow2=pow2)
        ctx.save_for_backward(qx_t, sx_t, qw_t, sw)
        ctx.pow2 = pow2
        ctx.weight = weight
        ctx.x_shape = x.shape
        return y.reshape(*x.shape[:-1], n)

    @staticmethod
    def backward(ctx, dy):
        qx_t, sx_t, qw_t, sw = ctx.saved_tensors
        weight = ctx.weight
        n, k = weight.shape
        dy2 = _rows(dy, n)
        qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy2, with_rowwise=True,
                                                      pow2=ctx.pow2)
        dx = dw = None
        if ctx.needs_input_grad[0]:
            dx = ops.gemm_dgrad(qdy, sdy, qw_t, sw, qw_is_transposed=True,
                                pow2=ctx.pow2).reshape(ctx.x_shape)
        if ctx.needs_input_grad[1]:
            main = getattr(weight, "main_grad", None)
            if main is not None:
                ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, main_grad=main,
                                   pow2=ctx.pow2)
            else:
                dw = ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, pow2=ctx.pow2)
                if dw.dtype != weight.dtype:
                    dw = dw.to(weight.dtype)
        return dx, dw, None


class BlockwiseFp8Linear(torch.nn.Module):
    """Bias-free linear layer (in_features -> out_features) whose three GEMMs
    run in blockwise E4M3. The weight is a bf16 parameter [out, in]; give it
    an fp32 `main_grad` tensor of the same shape to have dW accumulated there
    in fp32 instead of returned as `weight.grad`."""

    def __init__(self, in_features, out_features, device=None, pow2=False):
        super().__init__()
        if in_features % 16 or out_features % 16:
            raise ValueError("in_features and out_features must be multiples "
                             "of 16")
        self.in_features = in_features
        self.out_features = out_features
        self.pow2 = pow2
        w = torch.empty((out_features, in_features), dtype=torch.bfloat16,
                        device=device)
        torch.nn.init.normal_(w, std=0.02)
        self.weight = torch.nn.Parameter(w)

    def forward(self, x):
        return BlockwiseFp8LinearFunction.apply(x, self.weight, self.pow2)

    def extra_repr(self):
        return "in_features=%d, out_features=%d, pow2=%s" % (
            self.in_features, self.out_features, self.pow2)


class BlockwiseFp8ChainFunction(torch.autograd.Function):
    """y = x @ W_0.T @ W_1.T ... @ W_{L-1}.T: linears that feed one another
    directly, each on the blockwise-FP8 path, with every intermediate
    quantisation fused into the GEMM that produces it.

    Forward: the weights are block-quantised in batched launches (up to 8
    per launch); each fprop but the last also writes the row-wise (next
    fprop) and column-wise (next wgrad) codes of its bf16 output, so the next
    linear reads codes instead of re-reading and re-quantising the activation.
    Backward: each dgrad but the first linear's does the same for the
    gradient it produces, which is the previous linear's dY; the weight
    gradients, which all contract over the same tokens, are deferred to the
    end and computed in batched launches (up to 4 per launch). The results are
    those of the same linears run one by one (the fused codes are, bit for
    bit, those of quantising the bf16 output, and a batched launch computes
    what its jobs compute alone)."""

    @staticmethod
    def forward(ctx, x, *weights):
        k0 = weights[0].shape[1]
        h = _rows(x, k0)
        qx_t, sx_t, qx, sx = ops.quantize_colwise(h, with_rowwise=True)
        ws = [_rows(w, w.shape[1]) for w in weights]
        qws = []
        for j in range(0, len(ws), _WEIGHT_BATCH):
            qws += ops.quantize_weight_block_batch(ws[j:j + _WEIGHT_BATCH], transposed=True)
        saved = []
        y = None
        for i, (qw, sw, qw_t) in enumerate(qws):
            saved += [qx_t, sx_t, qw_t, sw]
            if i + 1 < len(weights):
                y, qx, sx, qx_t, sx_t = ops.gemm_fprop_quant_rowcol(qx, sx, qw, sw)
            else:
                y = ops.gemm_fprop(qx, sx, qw, sw)
        ctx.save_for_backward(*saved)
        ctx.weights = weights
        ctx.x_shape = x.shape
        return y.reshape(*x.shape[:-1], weights[-1].shape[0])

    @staticmethod
    def backward(ctx, dy):
        saved = ctx.saved_tensors
        weights = ctx.weights
        n_last = weights[-1].shape[0]
        dy2 = _rows(dy, n_last)
        qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy2, with_rowwise=True)
        grads = [None] * len(weights)
        dx = None
        to_main, to_grad = [], []      # deferred wgrads: (index, operands)
        for i in range(len(weights) - 1, -1, -1):
            qx_t, sx_t, qw_t, sw = saved[4 * i:4 * i + 4]
            if ctx.needs_input_grad[1 + i]:
                job = (i, (qdy_t, sdy_t, qx_t, sx_t))
                if getattr(weights[i], "main_grad", None) is not None:
                    to_main.append(job)
                else:
                    to_grad.append(job)
            if i > 0:
                _, qdy, sdy, qdy_t, sdy_t = ops.gemm_dgrad_quant_rowcol(
                    qdy, sdy, qw_t, sw, qw_is_transposed=True)
            elif ctx.needs_input_grad[0]:
                dx = ops.gemm_dgrad(qdy, sdy, qw_t, sw,
                                    qw_is_transposed=True).reshape(ctx.x_shape)
        for j in range(0, len(to_main), _WGRAD_BATCH):
            part = to_main[j:j + _WGRAD_BATCH]
            ops.gemm_wgrad_f32_batch([op for _, op in part],
                                     main_grads=[weights[i].main_grad for i, _ in part])
        for j in range(0, len(to_grad), _WGRAD_BATCH):
            part = to_grad[j:j + _WGRAD_BATCH]
            for (i, _), dw in zip(part, ops.gemm_wgrad_batch([op for _, op in part])):
                grads[i] = dw if dw.dtype == weights[i].dtype else dw.to(weights[i].dtype)
        return (dx, *grads)


class BlockwiseFp8Chain(torch.nn.Module):
    """Bias-free linears applied one after another with nothing in between
    (features[0] -> features[1] -> ... -> features[-1]), as
    BlockwiseFp8ChainFunction: the quantisation of every intermediate
    activation and gradient is fused into the GEMM that produces it."""

    def __init__(self, features, device=None):
        super().__init__()
        if len(features) < 2 or any(f % 16 for f in features):
            raise ValueError("need at least two feature sizes, each a multiple "
                             "of 16")
        self.features = list(features)
        ws = []
        for fin, fout in zip(features[:-1], features[1:]):
            w = torch.empty((fout, fin), dtype=torch.bfloat16, device=device)
            torch.nn.init.normal_(w, std=0.02)
            ws.append(torch.nn.Parameter(w))
        self.weights = torch.nn.ParameterList(ws)

    def forward(self, x):
        return BlockwiseFp8ChainFunction.apply(x, *self.weights)

    def extra_repr(self):
        return "features=%s" % (self.features,)


__all__ = ["BlockwiseFp8Linear", "BlockwiseFp8LinearFunction",
           "BlockwiseFp8Chain", "BlockwiseFp8ChainFunction"]
