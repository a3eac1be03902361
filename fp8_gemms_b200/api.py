"""Allocation helpers over the C ABI: PyTorch provides the device buffers,
libfp8lm.so does every step of the computation.

    from fp8_gemms_b200 import api
    mlp = api.Relu2Mlp(M, d, f)          # caller-owned saved tensors + workspace
    Y = mlp.forward(X, W_up, W_down)
    dX, dW_up, dW_down = mlp.backward(dY)

    lin = api.Linear(M, K, N)            # a plain linear Y = X W^T (attention, LM head)
    Y = lin.forward(X, W)
    dX, dW = lin.backward(dY)
"""
import torch

from . import _lib
from ._lib import (E4M3, E5M2, EPI_ACCUM_F32, EPI_NONE, EPI_RELU2_BWD,  # noqa: F401
                   EPI_RELU2_FWD, GEMM_A_MN_MAJOR, GEMM_B_MN_MAJOR, LINEAR_ACCUMULATE_WGRAD,
                   LINEAR_REUSE_WEIGHT_CAST, MLP_ACCUMULATE_WGRAD, MLP_REUSE_WEIGHT_CASTS,
                   LmError)


def _dev(t):
    return t.device


def new_scales(device, n=1):
    """n blocks of 4 fp32 {amax, scale, inv_scale, unused}, zeroed."""
    return torch.zeros(n, 4, dtype=torch.float32, device=device)


def cast(x, fmt, relu2_input=False, amax_in=None, want_q=True, want_qT=True, scales=None,
         stream=None):
    """Dynamic tensorwise cast of a bf16 [rows x cols] tensor.  Returns
    (q, qT, scales) with scales = [amax, scale, inv_scale, 0] on the device."""
    rows, cols = x.shape
    dev = _dev(x)
    q = torch.empty(rows, cols, dtype=torch.uint8, device=dev) if want_q else None
    qT = torch.empty(cols, rows, dtype=torch.uint8, device=dev) if want_qT else None
    sc = new_scales(dev)[0] if scales is None else scales
    _lib.lm_fp8_amax_scale_cast(x, fmt, sc[0:1], sc[1:2], sc[2:3], q, qT,
                                relu2_input=relu2_input, amax_in=amax_in, stream=stream)
    return q, qT, sc


def gemm_workspace(device="cuda"):
    """Scratch that lets a GEMM split its under-filled last wave of tiles."""
    return torch.empty(_lib.lm_fp8_gemm_workspace_size(), dtype=torch.uint8, device=device)


def gemm(A, fa, B, fb, inv_a, inv_b, epi=EPI_NONE, aux=None, amax_out=None, out=None,
         flags=0, workspace=None, stream=None):
    """bf16 D[M x N] = epi(A B^T inv_a inv_b) for FP8 codes A [M x K], B [N x K];
    with GEMM_A_MN_MAJOR / GEMM_B_MN_MAJOR in flags, A is given as [K x M] /
    B as [K x N] (the row-major codes of the transpose).  workspace: see
    gemm_workspace (None: no split-K tail)."""
    M = A.shape[1] if flags & GEMM_A_MN_MAJOR else A.shape[0]
    N = B.shape[1] if flags & GEMM_B_MN_MAJOR else B.shape[0]
    D = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=_dev(A))
    _lib.lm_fp8_gemm_ex(A, fa, B, fb, inv_a, inv_b, D, flags=flags, epi=epi, aux=aux,
                        amax_out=amax_out, workspace=workspace, stream=stream)
    return D


class Relu2Mlp:
    """Buffers for one relu^2 MLP block of shape (M, d, f): the forward's saved
    tensors (one device allocation carved by the library) and the backward's
    workspace.  forward()/backward() are single C-ABI calls."""

    def __init__(self, M, d, f, device="cuda"):
        self.M, self.d, self.f = M, d, f
        nbytes = _lib.lm_relu2_mlp_saved_bytes(M, d, f)
        if nbytes == 0:
            raise LmError(3, "lm_relu2_mlp_saved_bytes")
        self.saved_buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.saved = _lib.lm_relu2_mlp_saved_carve(self.saved_buf, M, d, f)
        self.workspace = torch.empty(_lib.lm_relu2_mlp_workspace_size(M, d, f),
                                     dtype=torch.uint8, device=device)
        self.device = device

    def forward(self, X, W_up, W_down, Y=None, stream=None, reuse_weight_casts=False):
        """reuse_weight_casts: W_up/W_down were cast by an earlier forward of
        the same weights (gradient accumulation); their casts are skipped."""
        if Y is None:
            Y = torch.empty(self.M, self.d, dtype=torch.bfloat16, device=self.device)
        if reuse_weight_casts:
            _lib.lm_relu2_mlp_fwd_ex(X, None, None, Y, self.saved, self.f,
                                     flags=MLP_REUSE_WEIGHT_CASTS, workspace=self.workspace,
                                     stream=stream)
        else:
            _lib.lm_relu2_mlp_fwd(X, W_up, W_down, Y, self.saved, workspace=self.workspace,
                                  stream=stream)
        return Y

    def backward_accumulate(self, dY, dW_up_f32, dW_down_f32, dX=None, stream=None):
        """Backward that adds this micro-batch's weight gradients into fp32
        accumulators dW_up_f32 [f x d] and dW_down_f32 [d x f]; returns dX."""
        dX = dX if dX is not None else torch.empty(self.M, self.d, dtype=torch.bfloat16,
                                                   device=self.device)
        assert dW_up_f32.dtype == torch.float32 and dW_down_f32.dtype == torch.float32
        _lib.lm_relu2_mlp_bwd_ex(dY, self.saved, dX, dW_up_f32, dW_down_f32, self.workspace,
                                 flags=MLP_ACCUMULATE_WGRAD, stream=stream)
        return dX

    def backward(self, dY, dX=None, dW_up=None, dW_down=None, stream=None):
        dev = self.device
        dX = dX if dX is not None else torch.empty(self.M, self.d, dtype=torch.bfloat16, device=dev)
        dW_up = dW_up if dW_up is not None else torch.empty(self.f, self.d, dtype=torch.bfloat16,
                                                            device=dev)
        dW_down = dW_down if dW_down is not None else torch.empty(self.d, self.f,
                                                                  dtype=torch.bfloat16, device=dev)
        _lib.lm_relu2_mlp_bwd(dY, self.saved, dX, dW_up, dW_down, self.workspace, stream=stream)
        return dX, dW_up, dW_down

    # views of the saved tensors (for inspection and stagewise checks)
    def view(self, name):
        M, d, f = self.M, self.d, self.f
        shapes = {"Xq": (M, d), "Wuq": (f, d), "Wdq": (d, f), "hq": (M, f)}
        base = self.saved_buf.data_ptr()
        if name == "H":
            off = self.saved.H - base
            return self.saved_buf[off:off + M * f * 2].view(torch.bfloat16).view(M, f)
        if name == "scales":
            off = self.saved.scales - base
            return self.saved_buf[off:off + 64].view(torch.float32).view(4, 4)
        r, c = shapes[name]
        off = getattr(self.saved, name) - base
        return self.saved_buf[off:off + r * c].view(r, c)

    def workspace_view(self, name):
        """Backward scratch: the GEMMs' split-K scratch, then dYq, dH, dHq,
        scales (library layout: each buffer rounded up to 256 bytes)."""
        M, d, f = self.M, self.d, self.f
        r256 = lambda n: (n + 255) // 256 * 256
        sizes = [("split", _lib.lm_fp8_gemm_workspace_size()), ("dYq", M * d),
                 ("dH", M * f * 2), ("dHq", M * f), ("scales", 32)]
        off = 0
        for n, sz in sizes:
            if n == name:
                v = self.workspace[off:off + sz]
                if n == "dH":
                    return v.view(torch.bfloat16).view(M, f)
                if n == "scales":
                    return v.view(torch.float32).view(2, 4)
                return v.view(*{"dYq": (M, d), "dHq": (M, f)}[n])
            off += r256(sz)
        raise KeyError(name)


def interleave_gate_up(W_gate, W_up):
    """[2f x d] weight whose rows alternate 128-row blocks of W_gate and W_up
    (the layout the gated MLP's single up GEMM reads)."""
    f, d = W_gate.shape
    assert f % 128 == 0 and W_up.shape == (f, d)
    return torch.stack([W_gate.view(f // 128, 128, d), W_up.view(f // 128, 128, d)],
                       dim=1).reshape(2 * f, d)


def deinterleave_gate_up(W_gu):
    f2, d = W_gu.shape
    v = W_gu.view(f2 // 256, 2, 128, d)
    return v[:, 0].reshape(f2 // 2, d), v[:, 1].reshape(f2 // 2, d)


class SwigluMlp:
    """Buffers of one gated (SwiGLU) MLP block (M, d, f) over the C ABI."""

    def __init__(self, M, d, f, device="cuda"):
        self.M, self.d, self.f = M, d, f
        nbytes = _lib.lib.lm_swiglu_mlp_saved_bytes(M, d, f)
        if nbytes == 0:
            raise LmError(3, "lm_swiglu_mlp_saved_bytes")
        self.saved_buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.saved = _lib.lm_swiglu_mlp_saved_carve(self.saved_buf, M, d, f)
        self.workspace = torch.empty(_lib.lib.lm_swiglu_mlp_workspace_size(M, d, f),
                                     dtype=torch.uint8, device=device)
        self.device = device

    def forward(self, X, W_gu, W_down, Y=None, stream=None):
        Y = Y if Y is not None else torch.empty(self.M, self.d, dtype=torch.bfloat16,
                                                device=self.device)
        _lib.lm_swiglu_mlp_fwd(X, W_gu, W_down, Y, self.saved, workspace=self.workspace,
                               stream=stream)
        return Y

    def backward(self, dY, dX=None, dW_gu=None, dW_down=None, stream=None):
        dev, M, d, f = self.device, self.M, self.d, self.f
        dX = dX if dX is not None else torch.empty(M, d, dtype=torch.bfloat16, device=dev)
        dW_gu = dW_gu if dW_gu is not None else torch.empty(2 * f, d, dtype=torch.bfloat16,
                                                            device=dev)
        dW_down = dW_down if dW_down is not None else torch.empty(d, f, dtype=torch.bfloat16,
                                                                  device=dev)
        _lib.lm_swiglu_mlp_bwd(dY, self.saved, dX, dW_gu, dW_down, self.workspace, stream=stream)
        return dX, dW_gu, dW_down

    def view(self, name):
        """Saved tensors: Xq, Wguq, Wdq, GU, h, hq, scales (library layout)."""
        M, d, f = self.M, self.d, self.f
        base = self.saved_buf.data_ptr()
        off = getattr(self.saved, name) - base
        if name in ("GU", "h"):
            cols = 2 * f if name == "GU" else f
            return self.saved_buf[off:off + M * cols * 2].view(torch.bfloat16).view(M, cols)
        if name == "scales":
            return self.saved_buf[off:off + 64].view(torch.float32).view(4, 4)
        shape = {"Xq": (M, d), "Wguq": (2 * f, d), "Wdq": (d, f), "hq": (M, f)}[name]
        return self.saved_buf[off:off + shape[0] * shape[1]].view(*shape)


class LmHeadCE:
    """Workspace of the chunked FP8 LM head with softcapped cross-entropy."""

    def __init__(self, M, d, V, chunk, device="cuda"):
        self.M, self.d, self.V, self.chunk = M, d, V, chunk
        n = _lib.lib.lm_fp8_lmhead_ce_workspace_size(M, d, V, chunk)
        if n == 0:
            raise LmError(3, "lm_fp8_lmhead_ce_workspace_size")
        self.workspace = torch.empty(n, dtype=torch.uint8, device=device)
        self.loss = torch.zeros(1, dtype=torch.float32, device=device)
        self.device = device

    def __call__(self, X, W, labels, dW=None, dX=None, softcap=15.0, stream=None):
        """Mean loss (device scalar), dX (bf16) and dW (fp32, accumulated)."""
        dX = dX if dX is not None else torch.empty_like(X)
        dW = dW if dW is not None else torch.zeros(self.V, self.d, dtype=torch.float32,
                                                   device=self.device)
        _lib.lm_fp8_lmhead_ce(X, W, labels, self.loss, dX, dW, self.workspace, self.chunk,
                              softcap=softcap, stream=stream)
        return self.loss, dX, dW

    def row_losses(self):
        """Per-token losses of the last call (the workspace's tail)."""
        n = self.M * 4
        tail = (n + 255) // 256 * 256
        return self.workspace[-tail:][:n].view(torch.float32)

    def view(self, name):
        """Workspace views after a call (library layout, each part rounded up
        to 256 bytes): "scales" [3 x 4] {amax, scale, inv_scale, 0} of X, W and
        the last chunk's dlogits; "Wq" [V x d]; and the last chunk's "Xq"
        [C x d], "dlogits" (bf16, written over its logits) [C x V] and "dLq"
        [C x V], where C is that chunk's row count."""
        M, d, V, C = self.M, self.d, self.V, self.chunk
        r256 = lambda n: (n + 255) // 256 * 256
        rows = M - (M - 1) // C * C if M else 0
        off = {"scales": 0}
        off["Wq"] = r256(64)
        off["Xq"] = off["Wq"] + r256(V * d)
        off["dlogits"] = off["Xq"] + r256(C * d)
        off["dLq"] = off["dlogits"] + r256(C * V * 2)
        o = off[name]
        ws = self.workspace
        if name == "scales":
            return ws[o:o + 48].view(torch.float32).view(3, 4)
        if name == "Wq":
            return ws[o:o + V * d].view(V, d)
        if name == "Xq":
            return ws[o:o + rows * d].view(rows, d)
        if name == "dlogits":
            return ws[o:o + rows * V * 2].view(torch.bfloat16).view(rows, V)
        return ws[o:o + rows * V].view(rows, V)


class Linear:
    """Buffers of one plain FP8 linear Y = X W^T with X [M x K], W [N x K]:
    the forward's saved codes and scales (one device allocation carved by the
    library) and the backward's workspace.  forward()/backward() are single
    C-ABI calls."""

    def __init__(self, M, K, N, device="cuda"):
        self.M, self.K, self.N = M, K, N
        nbytes = _lib.lm_fp8_linear_saved_bytes(M, K, N)
        if nbytes == 0:
            raise LmError(3, "lm_fp8_linear_saved_bytes")
        self.saved_buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.saved = _lib.lm_fp8_linear_saved_carve(self.saved_buf, M, K, N)
        self.workspace = torch.empty(_lib.lm_fp8_linear_workspace_size(M, K, N),
                                     dtype=torch.uint8, device=device)
        self.device = device

    def forward(self, X, W, Y=None, stream=None, reuse_weight_cast=False):
        if Y is None:
            Y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=self.device)
        _lib.lm_fp8_linear_fwd(X, None if reuse_weight_cast else W, Y, self.saved, self.N,
                               flags=LINEAR_REUSE_WEIGHT_CAST if reuse_weight_cast else 0,
                               workspace=self.workspace, stream=stream)
        return Y

    def backward(self, dY, dX=None, dW=None, need_dX=True, stream=None):
        """Returns (dX, dW); dX is None when need_dX is False (no dgrad)."""
        dev = self.device
        if need_dX and dX is None:
            dX = torch.empty(self.M, self.K, dtype=torch.bfloat16, device=dev)
        if dW is None:
            dW = torch.empty(self.N, self.K, dtype=torch.bfloat16, device=dev)
        _lib.lm_fp8_linear_bwd(dY, self.saved, self.K, dX if need_dX else None, dW,
                               self.workspace, stream=stream)
        return (dX if need_dX else None), dW

    def backward_accumulate(self, dY, dW_f32, dX=None, need_dX=True, stream=None):
        """Backward that adds this call's weight gradient into the fp32
        accumulator dW_f32 [N x K]; returns dX (None when need_dX is False)."""
        assert dW_f32.dtype == torch.float32
        if need_dX and dX is None:
            dX = torch.empty(self.M, self.K, dtype=torch.bfloat16, device=self.device)
        _lib.lm_fp8_linear_bwd(dY, self.saved, self.K, dX if need_dX else None, dW_f32,
                               self.workspace, flags=LINEAR_ACCUMULATE_WGRAD, stream=stream)
        return dX if need_dX else None

    # views of the saved and scratch buffers (for inspection and stagewise checks)
    def view(self, name):
        M, K, N = self.M, self.K, self.N
        base = self.saved_buf.data_ptr()
        off = getattr(self.saved, name) - base
        if name == "scales":
            return self.saved_buf[off:off + 32].view(torch.float32).view(2, 4)
        r, c = {"Xq": (M, K), "Wq": (N, K)}[name]
        return self.saved_buf[off:off + r * c].view(r, c)

    def workspace_view(self, name):
        """Backward scratch (library layout, each part rounded up to 256
        bytes): the GEMMs' split-K scratch, dY's codes, dY's scale block."""
        r256 = lambda n: (n + 255) // 256 * 256
        off = r256(_lib.lm_fp8_gemm_workspace_size())
        n = self.M * self.N
        if name == "dYq":
            return self.workspace[off:off + n].view(self.M, self.N)
        if name == "scales":
            off += r256(n)
            return self.workspace[off:off + 16].view(torch.float32)
        raise KeyError(name)


def linear_fwd_bwd(X, W, dY, stream=None):
    """Plain linear Y = X W^T with its dgrad and wgrad, all in FP8, through
    lm_fp8_linear_fwd and lm_fp8_linear_bwd: X, W cast to e4m3 and dY to e5m2
    (row-major codes only), then Y = Xq Wq^T, dX = dYq W (Wq read MN-major),
    dW = dY^T X (dYq and Xq read MN-major).
    Returns (Y, dX, dW, intermediates): the codes Xq, Wq, dYq and a [3 x 4]
    host array of the {amax, scale, inv_scale, 0} blocks of X, W and dY."""
    M, K = X.shape
    N = W.shape[0]
    lin = Linear(M, K, N, device=X.device)
    Y = lin.forward(X, W, stream=stream)
    dX, dW = lin.backward(dY, stream=stream)
    if stream is not None:
        stream.synchronize()
    sc = torch.cat([lin.view("scales"), lin.workspace_view("scales").view(1, 4)]).cpu().numpy()
    return Y, dX, dW, dict(Xq=lin.view("Xq"), Wq=lin.view("Wq"), dYq=lin.workspace_view("dYq"),
                           scales=sc)
