"""ctypes binding of libomq (include/omq.h): argument marshalling only.

PyTorch tensors supply device memory and the current stream; every computation runs in the
library's CUDA kernels. Importing this module loads ``libomq.so`` from the package
directory and raises ImportError when it is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libomq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libomq.so is not built ({LIB_PATH}); run "
                      "`python -m post_quantization_lwc_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

OMQ_F32, OMQ_BF16, OMQ_F16 = 0, 1, 2
STATUS = {0: "OMQ_OK", 1: "OMQ_ERR_NULL", 2: "OMQ_ERR_SHAPE", 3: "OMQ_ERR_DTYPE",
          4: "OMQ_ERR_ALIGN", 5: "OMQ_ERR_BITS", 6: "OMQ_ERR_WORKSPACE", 7: "OMQ_ERR_CUDA",
          8: "OMQ_ERR_UNSUPPORTED", 9: "OMQ_ERR_TIMEOUT"}

# every symbol declared in include/omq.h
EXPORTS = ("omq_status_str", "omq_last_cuda_error", "omq_version", "omq_sync_check",
           "omq_lwc_quant", "omq_let_apply", "omq_fq_linear_fwd", "omq_fwd_workspace_bytes",
           "omq_fq_linear_bwd", "omq_bwd_workspace_bytes", "omq_adamw_step", "omq_fold_pack",
           "omq_calib_step", "omq_step_workspace_bytes", "omq_launch_count",
           "omq_fq_linear_fwd_noalloc", "omq_block_theta_range", "omq_block_buffer",
           "omq_block_workspace_bytes", "omq_block_step", "omq_block_reference",
           "omq_block_quant_forward", "omq_block_calibrate", "omq_qgemv",
           "omq_set_wait_limit_ns", "omq_wait_limit_ns", "omq_wait_probe", "omq_qgemm")

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_f32 = ctypes.c_float
_sz = ctypes.c_size_t


class OmqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.omq_status_str(status).decode()
        extra = f" (cuda error {_lib.omq_last_cuda_error()})" if status == 7 else ""
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}{extra}")


class BwdArgs(ctypes.Structure):
    _fields_ = [("M", _i64), ("N", _i64), ("K", _i64), ("group", _i64), ("bits", _i32),
                ("abits", _i32), ("dt", _i32), ("op_dt", _i32),
                ("X", _p), ("W", _p), ("s", _p), ("delta", _p), ("gamma_logit", _p),
                ("beta_logit", _p), ("Xq", _p), ("W_hat", _p), ("h", _p), ("z", _p),
                ("grp_range", _p), ("h_a", _p), ("z_a", _p), ("tok_range", _p), ("dY", _p),
                ("d_gamma_logit", _p), ("d_beta_logit", _p), ("d_s", _p), ("d_delta", _p),
                ("d_B_tilde", _p)]


class StepArgs(ctypes.Structure):
    _fields_ = [("M", _i64), ("N", _i64), ("K", _i64), ("group", _i64), ("bits", _i32),
                ("abits", _i32), ("let", _i32), ("dt", _i32), ("op_dt", _i32),
                ("X", _p), ("W", _p), ("B", _p), ("Y_ref", _p),
                ("gamma_logit", _p), ("beta_logit", _p), ("s", _p), ("delta", _p),
                ("m_gamma", _p), ("v_gamma", _p), ("m_beta", _p), ("v_beta", _p),
                ("m_s", _p), ("v_s", _p), ("m_delta", _p), ("v_delta", _p),
                ("Xq", _p), ("W_hat", _p), ("B_tilde", _p),
                ("h", _p), ("z", _p), ("grp_range", _p),
                ("h_a", _p), ("z_a", _p), ("tok_range", _p),
                ("dY", _p),
                ("d_gamma_logit", _p), ("d_beta_logit", _p), ("d_s", _p), ("d_delta", _p),
                ("loss", _p), ("lr_lwc", _f32), ("lr_let", _f32), ("step", _i64),
                ("events", _p)]


class BlockDims(ctypes.Structure):
    _fields_ = [("M", _i64), ("D", _i64), ("H", _i64), ("I", _i64), ("group", _i64),
                ("wbits", _i32), ("abits", _i32)]


class BlockArgs(ctypes.Structure):
    _fields_ = [("dims", BlockDims), ("x", _p), ("y_ref", _p), ("W_qkv", _p), ("W_o", _p),
                ("W_gu", _p), ("W_d", _p), ("theta", _p), ("d_theta", _p), ("loss", _p),
                ("adam_m", _p), ("adam_v", _p), ("step", _i64), ("lr_lwc", _f32),
                ("lr_let", _f32), ("events", _p)]


class BlockCalibArgs(ctypes.Structure):
    _fields_ = [("dims", BlockDims), ("xs", _p), ("y_refs", _p), ("n_samples", _i64),
                ("epochs", _i64), ("W_qkv", _p), ("W_o", _p), ("W_gu", _p), ("W_d", _p),
                ("theta", _p), ("d_theta", _p), ("adam_m", _p), ("adam_v", _p),
                ("first_step", _i64), ("lr_lwc", _f32), ("lr_let", _f32), ("losses", _p)]


# phases of omq_calib_step (OMQ_PH_* in include/omq.h), in order
PHASES = ("let", "lwc", "fwd_gemm", "loss", "dbias", "dw_gemm", "ste_w", "dx_gemm", "ste_x",
          "let_reduce", "adamw")


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args


_sig("omq_status_str", ctypes.c_char_p, [_i32])
_sig("omq_last_cuda_error", _i32, [])
_sig("omq_version", _i32, [])
_sig("omq_sync_check", _i32, [_p])
_sig("omq_lwc_quant", _i32, [_p, _i32, _i64, _i64, _i64, _i32, _p, _p, _p, _p, _i32, _p, _p, _p,
                             _p, _p])
_sig("omq_let_apply", _i32, [_p, _i32, _i64, _i64, _p, _p, _i32, _p, _i32, _p, _p, _p, _p, _i32,
                             _i64, _p, _p, _p])
_sig("omq_fq_linear_fwd", _i32, [_p, _p, _i32, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _sz, _p])
_sig("omq_fwd_workspace_bytes", _sz, [_i64, _i64, _i64])
_sig("omq_fq_linear_bwd", _i32, [ctypes.POINTER(BwdArgs), _p, _sz, _p])
_sig("omq_bwd_workspace_bytes", _sz, [_i64, _i64, _i64, _i64])
_sig("omq_adamw_step", _i32, [_p, _p, _p, _p, _i64, _f32, _f32, _f32, _f32, _f32, _i64, _p])
_sig("omq_fold_pack", _i32, [_p, _i32, _i64, _i64, _i64, _i32, _p, _p, _p, _p, _p, _p, _p])
_sig("omq_calib_step", _i32, [ctypes.POINTER(StepArgs), _p, _sz, _p])
_sig("omq_step_workspace_bytes", _sz, [_i64, _i64, _i64, _i64])
_sig("omq_launch_count", ctypes.c_uint64, [])
_sig("omq_fq_linear_fwd_noalloc", _i32, [_p, _p, _i32, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p])
_sig("omq_block_theta_range", _i32, [ctypes.POINTER(BlockDims), _i32, ctypes.POINTER(_i64),
                                     ctypes.POINTER(_i64)])
_sig("omq_block_buffer", _i32, [ctypes.POINTER(BlockDims), _i32, ctypes.POINTER(_sz),
                                ctypes.POINTER(_sz)])
_sig("omq_block_workspace_bytes", _sz, [ctypes.POINTER(BlockDims)])
_sig("omq_block_step", _i32, [ctypes.POINTER(BlockArgs), _p, _sz, _p])
_sig("omq_block_reference", _i32, [ctypes.POINTER(BlockDims), _p, _p, _p, _p, _p, _p, _p, _sz,
                                   _p])
_sig("omq_block_quant_forward", _i32, [ctypes.POINTER(BlockDims), _p, _p, _p, _p, _p, _p, _p,
                                       _i32, _p, _sz, _p])
_sig("omq_block_calibrate", _i32, [ctypes.POINTER(BlockCalibArgs), _p, _sz, _p])
_sig("omq_qgemv", _i32, [_p, _i32, _i64, _i64, _p, _p, _p, _i64, _i64, _i32, _p, _p])
_sig("omq_set_wait_limit_ns", _i32, [ctypes.c_uint64])
_sig("omq_wait_limit_ns", ctypes.c_uint64, [])
_sig("omq_wait_probe", _i32, [_i32, _p])
_sig("omq_qgemm", _i32, [_p, _i32, _i64, _i64, _p, _p, _p, _i64, _i64, _i32, _p, _p, _p])


def _check(status: int, where: str):
    if status != 0:
        raise OmqError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_DTYPES = {torch.float32: OMQ_F32, torch.bfloat16: OMQ_BF16, torch.float16: OMQ_F16}


def _dt(t) -> int:
    dtype = t if isinstance(t, torch.dtype) else t.dtype
    if dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {dtype}")
    return _DTYPES[dtype]


def operand_dtype(storage: torch.dtype, act_pass: bool = True) -> torch.dtype:
    """GEMM operand dtype the step uses for a storage dtype: float32 for float32 storage;
    for 16-bit storage float16 (3 more mantissa bits than bfloat16 at the same tensor-core
    rate) when the step writes its own activation operand anyway (LET or activation
    quantization, ``act_pass``), else the storage type itself, so that X is the operand as
    it stands and no conversion pass over it runs."""
    if storage == torch.float32:
        return torch.float32
    return torch.float16 if act_pass else storage


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def version() -> int:
    return _lib.omq_version()


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.omq_launch_count())


def sync_check(stream=None):
    _check(_lib.omq_sync_check(_stream(stream)), "omq_sync_check")


def set_wait_limit_ns(ns: int):
    _check(_lib.omq_set_wait_limit_ns(ctypes.c_uint64(int(ns))), "omq_set_wait_limit_ns")


def wait_limit_ns() -> int:
    return int(_lib.omq_wait_limit_ns())


def wait_probe(arrive: bool, stream=None):
    _check(_lib.omq_wait_probe(1 if arrive else 0, _stream(stream)), "omq_wait_probe")


def new_range(n: int, device) -> torch.Tensor:
    """Storage for omq_range records (16 bytes each) as an int32 [n, 4] tensor."""
    return torch.empty(n, 4, dtype=torch.int32, device=device)


def range_fields(r: torch.Tensor):
    """(vmax, vmin, nmax, nmin) views of an omq_range tensor."""
    return r[:, 0].view(torch.float32), r[:, 1].view(torch.float32), r[:, 2], r[:, 3]


# ---------------------------------------------------------------------------- primitives

def lwc_quant(W, gamma_logit, beta_logit, bits, group, s=None, hat_dtype=None, codes=False,
              stream=None):
    """omq_lwc_quant. Returns dict(W_hat, h, z, codes, grp_range)."""
    _dev(W, gamma_logit, beta_logit, s)
    N, K = W.shape
    ng = K // group
    dev = W.device
    W_hat = torch.empty(N, K, dtype=hat_dtype or W.dtype, device=dev)
    h = torch.empty(N, ng, dtype=torch.float32, device=dev)
    z = torch.empty(N, ng, dtype=torch.int32, device=dev)
    c = torch.empty(N, K, dtype=torch.uint8, device=dev) if codes else None
    rg = new_range(N * ng, dev)
    _check(_lib.omq_lwc_quant(_ptr(W), _dt(W), N, K, group, bits, _ptr(gamma_logit),
                              _ptr(beta_logit), _ptr(s), _ptr(W_hat), _dt(W_hat), _ptr(h), _ptr(z),
                              _ptr(c), _ptr(rg), _stream(stream)), "omq_lwc_quant")
    return dict(W_hat=W_hat, h=h, z=z, codes=c, grp_range=rg)


def let_apply(X, abits, s=None, delta=None, xq_dtype=None, W=None, B=None, want_bias=False,
              stream=None):
    """omq_let_apply. Returns dict(Xq, h_a, z_a, tok_range, B_tilde)."""
    _dev(X, s, delta, W, B)
    M, K = X.shape
    dev = X.device
    Xq = torch.empty(M, K, dtype=xq_dtype or X.dtype, device=dev)
    q = abits < 16
    h_a = torch.empty(M, dtype=torch.float32, device=dev) if q else None
    z_a = torch.empty(M, dtype=torch.int32, device=dev) if q else None
    tr = new_range(M, dev) if q else None
    N = W.shape[0] if W is not None else (B.shape[0] if B is not None else 0)
    Bt = torch.empty(N, dtype=torch.float32, device=dev) if want_bias else None
    _check(_lib.omq_let_apply(_ptr(X), _dt(X), M, K, _ptr(s), _ptr(delta), abits, _ptr(Xq),
                              _dt(Xq), _ptr(h_a), _ptr(z_a), _ptr(tr), _ptr(W),
                              _dt(W) if W is not None else 0, N, _ptr(B), _ptr(Bt),
                              _stream(stream)), "omq_let_apply")
    return dict(Xq=Xq, h_a=h_a, z_a=z_a, tok_range=tr, B_tilde=Bt)


def fwd_workspace_bytes(M, N, K) -> int:
    return _lib.omq_fwd_workspace_bytes(M, N, K)


def fq_linear_fwd(Xq, W_hat, B_tilde=None, Y_ref=None, want_Y=True, workspace=None,
                  stream=None):
    """omq_fq_linear_fwd. Returns dict(Y, dY, loss)."""
    _dev(Xq, W_hat, B_tilde, Y_ref)
    M, K = Xq.shape
    N = W_hat.shape[0]
    dev = Xq.device
    Y = torch.empty(M, N, dtype=torch.float32, device=dev) if (want_Y or Y_ref is None) else None
    dY = torch.empty(M, N, dtype=Xq.dtype, device=dev) if Y_ref is not None else None
    loss = torch.empty(1, dtype=torch.float32, device=dev) if Y_ref is not None else None
    nbytes = fwd_workspace_bytes(M, N, K)
    if workspace is None and Y_ref is not None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(_lib.omq_fq_linear_fwd(_ptr(Xq), _ptr(W_hat), _dt(Xq), M, N, K, _ptr(B_tilde),
                                  _ptr(Y_ref), _ptr(Y), _ptr(dY), _ptr(loss), _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream)),
           "omq_fq_linear_fwd")
    return dict(Y=Y, dY=dY, loss=loss)


def fq_linear_fwd_noalloc(Xq, W_hat, Y_ref, B_tilde=None, want_Y=True, stream=None):
    """omq_fq_linear_fwd_noalloc: the forward with its loss for hosts that cannot lend the
    library device scratch; the scratch is a fixed array inside the library (see omq.h).
    Returns dict(Y, dY, loss)."""
    _dev(Xq, W_hat, B_tilde, Y_ref)
    M, K = Xq.shape
    N = W_hat.shape[0]
    dev = Xq.device
    Y = torch.empty(M, N, dtype=torch.float32, device=dev) if want_Y else None
    dY = torch.empty(M, N, dtype=Xq.dtype, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    _check(_lib.omq_fq_linear_fwd_noalloc(_ptr(Xq), _ptr(W_hat), _dt(Xq), M, N, K, _ptr(B_tilde),
                                          _ptr(Y_ref), _ptr(Y), _ptr(dY), _ptr(loss),
                                          _stream(stream)), "omq_fq_linear_fwd_noalloc")
    return dict(Y=Y, dY=dY, loss=loss)


def bwd_workspace_bytes(M, N, K, group) -> int:
    return _lib.omq_bwd_workspace_bytes(M, N, K, group)


def fq_linear_bwd(*, X, W, gamma_logit, beta_logit, Xq, W_hat, h, z, grp_range, dY, bits, group,
                  abits=16, s=None, delta=None, h_a=None, z_a=None, tok_range=None,
                  want_let=False, want_dBt=False, workspace=None, stream=None):
    """omq_fq_linear_bwd. Returns dict(d_gamma_logit, d_beta_logit, d_s, d_delta, d_B_tilde)."""
    _dev(X, W, gamma_logit, beta_logit, Xq, W_hat, h, z, grp_range, dY, s, delta)
    M, K = Xq.shape
    N = W.shape[0]
    dev = W.device
    f = lambda *shape: torch.empty(*shape, dtype=torch.float32, device=dev)
    out = dict(d_gamma_logit=f(N, K // group), d_beta_logit=f(N, K // group),
               d_s=f(K) if want_let else None, d_delta=f(K) if want_let else None,
               d_B_tilde=f(N) if want_dBt else None)
    a = BwdArgs(M=M, N=N, K=K, group=group, bits=bits, abits=abits, dt=_dt(W), op_dt=_dt(Xq),
                X=_ptr(X), W=_ptr(W), s=_ptr(s), delta=_ptr(delta), gamma_logit=_ptr(gamma_logit),
                beta_logit=_ptr(beta_logit), Xq=_ptr(Xq), W_hat=_ptr(W_hat), h=_ptr(h), z=_ptr(z),
                grp_range=_ptr(grp_range), h_a=_ptr(h_a), z_a=_ptr(z_a), tok_range=_ptr(tok_range),
                dY=_ptr(dY), d_gamma_logit=_ptr(out["d_gamma_logit"]),
                d_beta_logit=_ptr(out["d_beta_logit"]), d_s=_ptr(out["d_s"]),
                d_delta=_ptr(out["d_delta"]), d_B_tilde=_ptr(out["d_B_tilde"]))
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(M, N, K, group), dtype=torch.uint8, device=dev)
    _check(_lib.omq_fq_linear_bwd(ctypes.byref(a), _ptr(workspace), workspace.numel(),
                                  _stream(stream)), "omq_fq_linear_bwd")
    return out


def adamw_step(param, grad, m, v, lr, step, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
               stream=None):
    """omq_adamw_step (in place on param, m, v)."""
    _dev(param, grad, m, v)
    _check(_lib.omq_adamw_step(_ptr(param), _ptr(grad), _ptr(m), _ptr(v), param.numel(), lr, beta1,
                               beta2, eps, weight_decay, step, _stream(stream)), "omq_adamw_step")


def fold_pack(W, gamma_logit, beta_logit, bits, group, s=None, stream=None):
    """omq_fold_pack. Returns (packed uint8 [N, K*bits/8], h, z)."""
    _dev(W, gamma_logit, beta_logit, s)
    N, K = W.shape
    dev = W.device
    packed = torch.empty(N, K * bits // 8, dtype=torch.uint8, device=dev)
    h = torch.empty(N, K // group, dtype=torch.float32, device=dev)
    z = torch.empty(N, K // group, dtype=torch.int32, device=dev)
    _check(_lib.omq_fold_pack(_ptr(W), _dt(W), N, K, group, bits, _ptr(gamma_logit),
                              _ptr(beta_logit), _ptr(s), _ptr(packed), _ptr(h), _ptr(z),
                              _stream(stream)), "omq_fold_pack")
    return packed, h, z


def qgemv(x, packed, h, z, group, bits, stream=None):
    """omq_qgemv: y [M, N] float32 = x dequant(packed, h, z)^T for 1..8 tokens."""
    _dev(x, packed, h, z)
    M, K = x.shape
    N = packed.shape[0]
    y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    _check(_lib.omq_qgemv(_ptr(x), _dt(x), M, K, _ptr(packed), _ptr(h), _ptr(z), N, group, bits,
                          _ptr(y), _stream(stream)), "omq_qgemv")
    return y


def qgemm(x, packed, h, z, group, bits, bias=None, stream=None):
    """omq_qgemm: y = x dequant(packed, h, z)^T (+ bias) on the tensor cores, any token count.
    x [M, K] float16 / bfloat16; returns y [M, N] float32."""
    _dev(x, packed, h, z, bias)
    M, K = x.shape
    N = packed.shape[0]
    y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    _check(_lib.omq_qgemm(_ptr(x), _dt(x), M, K, _ptr(packed), _ptr(h), _ptr(z), N, group, bits,
                          _ptr(bias), _ptr(y), _stream(stream)), "omq_qgemm")
    return y


def step_workspace_bytes(M, N, K, group) -> int:
    return _lib.omq_step_workspace_bytes(M, N, K, group)


# ---------------------------------------------------------------------------- whole step

@dataclasses.dataclass
class LinearCalibration:
    """Device buffers of one linear layer's calibration, driven by omq_calib_step.

    Holds W, the learnable parameters with their AdamW moments, the step's intermediate
    buffers and the workspace; ``step(X, Y_ref)`` runs one whole calibration step on the
    current stream (LET, LWC, forward + loss, STE backward, AdamW).
    """
    M: int
    N: int
    K: int
    group: int
    bits: int
    abits: int
    let: bool
    dtype: torch.dtype
    device: torch.device
    lr_lwc: float = 5e-3
    lr_let: float = 1e-2

    def __post_init__(self):
        dev, M, N, K = self.device, self.M, self.N, self.K
        ng = K // self.group
        f = lambda *shape: torch.zeros(*shape, dtype=torch.float32, device=dev)
        self.W = torch.empty(N, K, dtype=self.dtype, device=dev)
        self.B = f(N)
        self.gamma_logit, self.beta_logit = f(N, ng), f(N, ng)
        self.s, self.delta = f(K), f(K)
        self.moments = {k: (f(*shape), f(*shape)) for k, shape in
                        (("gamma", (N, ng)), ("beta", (N, ng)), ("s", (K,)), ("delta", (K,)))}
        self.op_dtype = operand_dtype(self.dtype, self.let or self.abits < 16)
        need_act = self.let or self.abits < 16 or self.op_dtype != self.dtype
        self.Xq = torch.empty(M, K, dtype=self.op_dtype, device=dev) if need_act else None
        self.W_hat = torch.empty(N, K, dtype=self.op_dtype, device=dev)
        self.B_tilde = f(N)
        self.h = f(N, ng)
        self.z = torch.zeros(N, ng, dtype=torch.int32, device=dev)
        self.grp_range = new_range(N * ng, dev)
        q = self.abits < 16
        self.h_a = f(M) if q else None
        self.z_a = torch.zeros(M, dtype=torch.int32, device=dev) if q else None
        self.tok_range = new_range(M, dev) if q else None
        self.dY = torch.empty(M, N, dtype=self.op_dtype, device=dev)
        self.d_gamma, self.d_beta = f(N, ng), f(N, ng)
        self.d_s, self.d_delta = f(K), f(K)
        self.loss = f(1)
        self.workspace = torch.empty(step_workspace_bytes(M, N, K, self.group), dtype=torch.uint8,
                                     device=dev)
        self.t = 0

    def load(self, W, gamma_logit, beta_logit, s=None, delta=None, B=None):
        self.W.copy_(W)
        self.gamma_logit.copy_(gamma_logit)
        self.beta_logit.copy_(beta_logit)
        if s is not None:
            self.s.copy_(s)
        if delta is not None:
            self.delta.copy_(delta)
        if B is not None:
            self.B.copy_(B)
        for m, v in self.moments.values():
            m.zero_()
            v.zero_()
        self.t = 0

    def args(self, X, Y_ref) -> StepArgs:
        mo = self.moments
        return StepArgs(
            M=self.M, N=self.N, K=self.K, group=self.group, bits=self.bits, abits=self.abits,
            let=1 if self.let else 0, dt=_dt(self.W), op_dt=_dt(self.op_dtype), X=_ptr(X),
            W=_ptr(self.W), B=_ptr(self.B),
            Y_ref=_ptr(Y_ref), gamma_logit=_ptr(self.gamma_logit), beta_logit=_ptr(self.beta_logit),
            s=_ptr(self.s), delta=_ptr(self.delta),
            m_gamma=_ptr(mo["gamma"][0]), v_gamma=_ptr(mo["gamma"][1]),
            m_beta=_ptr(mo["beta"][0]), v_beta=_ptr(mo["beta"][1]),
            m_s=_ptr(mo["s"][0]), v_s=_ptr(mo["s"][1]),
            m_delta=_ptr(mo["delta"][0]), v_delta=_ptr(mo["delta"][1]),
            Xq=_ptr(self.Xq), W_hat=_ptr(self.W_hat), B_tilde=_ptr(self.B_tilde), h=_ptr(self.h),
            z=_ptr(self.z), grp_range=_ptr(self.grp_range), h_a=_ptr(self.h_a), z_a=_ptr(self.z_a),
            tok_range=_ptr(self.tok_range), dY=_ptr(self.dY), d_gamma_logit=_ptr(self.d_gamma),
            d_beta_logit=_ptr(self.d_beta), d_s=_ptr(self.d_s), d_delta=_ptr(self.d_delta),
            loss=_ptr(self.loss), lr_lwc=self.lr_lwc, lr_let=self.lr_let, step=self.t)

    def step(self, X, Y_ref, stream=None, events=None):
        """One calibration step. ``events``: None, or len(PHASES) + 1 timing-enabled
        torch.cuda.Event objects recorded at the phase boundaries (see PhaseTimer)."""
        _dev(X, Y_ref)
        self.t += 1
        a = self.args(X, Y_ref)
        if events is not None:
            arr = (ctypes.c_void_p * (len(PHASES) + 1))(*[e.cuda_event for e in events])
            a.events = ctypes.cast(arr, ctypes.c_void_p)
        _check(_lib.omq_calib_step(ctypes.byref(a), _ptr(self.workspace), self.workspace.numel(),
                                   _stream(stream)), "omq_calib_step")
        return self.loss

    def reference_output(self, X, stream=None):
        """Y* = X W^T + B with the library's own GEMM (computed once, outside the step)."""
        return fq_linear_fwd(X, self.W, B_tilde=self.B, stream=stream)["Y"]


class PhaseTimer:
    """Per-step sets of CUDA events for omq_calib_step's phase boundaries."""

    def __init__(self, n_steps: int):
        self.sets = []
        for _ in range(n_steps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)]
            for e in evs:          # create the underlying cudaEvent_t now
                e.record()
            self.sets.append(evs)
        torch.cuda.synchronize()

    def mean_ms(self):
        """Average duration of each phase over the recorded steps (call after a sync)."""
        tot = [0.0] * len(PHASES)
        for evs in self.sets:
            for i in range(len(PHASES)):
                tot[i] += evs[i].elapsed_time(evs[i + 1])
        return {p: t / len(self.sets) for p, t in zip(PHASES, tot)}


# ---------------------------------------------------------------------------- transformer block

# theta tensors (OMQ_TH_* in include/omq.h) and workspace tensors (OMQ_BB_*), in order
THETA = ("gamma_qkv", "beta_qkv", "gamma_o", "beta_o", "gamma_gu", "beta_gu", "gamma_d",
         "beta_d", "s1", "delta1", "s_a", "s_o", "delta_o", "s2", "delta2")
# The block's named workspace tensors as omq_block_step leaves them: float16 GEMM operands,
# the gradients between stages unscaled (in units of the residual y - y*, i.e. gradients of
# (M D / 2) times the loss). omq_block_reference writes its 16-bit operands as bfloat16.
_H = torch.float16
BLOCK_BUFFERS = (
    ("rope", torch.float32), ("a", torch.float32), ("qa", _H),
    ("what_qkv", _H), ("what_o", _H), ("what_gu", _H),
    ("what_d", _H), ("qkv", torch.float32), ("qqkv", _H),
    ("p", torch.float32), ("p16", _H), ("o", torch.float32), ("qo", _H),
    ("x2", torch.float32), ("b", torch.float32), ("qb", _H), ("gu", torch.float32),
    ("mid", torch.float32), ("qm", _H), ("res", _H),
    ("dmid", torch.float32), ("dgu", _H), ("db", torch.float32),
    ("dx2", _H), ("do", _H), ("dqqkv", torch.float32),
    ("dqkv", _H))
BLOCK_PHASES = ("weights", "attn_in", "attn", "ffn", "bwd_ffn", "bwd_attn", "bwd_qkv", "reduce",
                "adamw")


class Block:
    """Device buffers of one transformer block's calibration, driven by omq_block_step.

    ``dims``: M tokens, D hidden (128 per head), H heads, I FFN size, LWC group (0 = per
    channel), wbits, abits. Holds the BF16 weights (W_qkv [3D, D], W_o [D, D], W_gu [2I, D],
    W_d [D, I]), the parameter vector theta with its gradient and AdamW moments, and the
    workspace whose tensors ``buffer(name)`` views.
    """

    def __init__(self, M, D, H, I, group=0, wbits=4, abits=4, device="cuda", lr_lwc=5e-3,
                 lr_let=1e-2):
        self.dims = BlockDims(M=M, D=D, H=H, I=I, group=group, wbits=wbits, abits=abits)
        self.device = torch.device(device)
        self.lr_lwc, self.lr_let = lr_lwc, lr_let
        nbytes = _lib.omq_block_workspace_bytes(ctypes.byref(self.dims))
        if nbytes == 0:
            raise ValueError("invalid block dimensions")
        off, cnt = _i64(), _i64()
        self.theta_slices = {}
        for i, name in enumerate(THETA):
            _check(_lib.omq_block_theta_range(ctypes.byref(self.dims), i, ctypes.byref(off),
                                              ctypes.byref(cnt)), "omq_block_theta_range")
            self.theta_slices[name] = (off.value, cnt.value)
        _check(_lib.omq_block_theta_range(ctypes.byref(self.dims), len(THETA), ctypes.byref(off),
                                          ctypes.byref(cnt)), "omq_block_theta_range")
        self.P = cnt.value
        f = lambda n: torch.zeros(n, dtype=torch.float32, device=self.device)  # noqa: E731
        self.theta, self.d_theta = f(self.P), f(self.P)
        self.adam_m, self.adam_v = f(self.P), f(self.P)
        self.loss = f(1)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        b = lambda *shape: torch.zeros(*shape, dtype=torch.bfloat16, device=self.device)  # noqa
        self.W = {"qkv": b(3 * D, D), "o": b(D, D), "gu": b(2 * I, D), "d": b(D, I)}
        self.t = 0

    def theta_part(self, name, t=None):
        o, n = self.theta_slices[name]
        return (self.theta if t is None else t)[o:o + n]

    def buffer(self, name):
        """The workspace tensor `name` (BLOCK_BUFFERS) as a flat tensor view."""
        idx = [n for n, _ in BLOCK_BUFFERS].index(name)
        dtype = BLOCK_BUFFERS[idx][1]
        off, nb = _sz(), _sz()
        _check(_lib.omq_block_buffer(ctypes.byref(self.dims), idx, ctypes.byref(off),
                                     ctypes.byref(nb)), "omq_block_buffer")
        esz = torch.empty(0, dtype=dtype).element_size()
        return self.workspace[off.value:off.value + nb.value].view(dtype)[: nb.value // esz]

    def load(self, W, theta):
        for k in self.W:
            self.W[k].copy_(W[k])
        self.theta.copy_(theta)
        self.adam_m.zero_()
        self.adam_v.zero_()
        self.t = 0

    def reference(self, x, out=None, stream=None):
        """omq_block_reference: the full-precision block output y* [M, D] float32 (written
        into `out` when given)."""
        _dev(x, out)
        y = out if out is not None else torch.empty(self.dims.M, self.dims.D,
                                                    dtype=torch.float32, device=self.device)
        _check(_lib.omq_block_reference(ctypes.byref(self.dims), _ptr(x), _ptr(self.W["qkv"]),
                                        _ptr(self.W["o"]), _ptr(self.W["gu"]), _ptr(self.W["d"]),
                                        _ptr(y), _ptr(self.workspace), self.workspace.numel(),
                                        _stream(stream)), "omq_block_reference")
        return y

    def step(self, x, y_ref, update=True, stream=None, events=None):
        """omq_block_step: forward, loss, backward (d_theta) and, with update, AdamW."""
        _dev(x, y_ref)
        if update:
            self.t += 1
        a = BlockArgs(dims=self.dims, x=_ptr(x), y_ref=_ptr(y_ref), W_qkv=_ptr(self.W["qkv"]),
                      W_o=_ptr(self.W["o"]), W_gu=_ptr(self.W["gu"]), W_d=_ptr(self.W["d"]),
                      theta=_ptr(self.theta), d_theta=_ptr(self.d_theta), loss=_ptr(self.loss),
                      adam_m=_ptr(self.adam_m) if update else None,
                      adam_v=_ptr(self.adam_v) if update else None, step=max(self.t, 1),
                      lr_lwc=self.lr_lwc, lr_let=self.lr_let)
        if events is not None:
            arr = (ctypes.c_void_p * (len(BLOCK_PHASES) + 1))(*[e.cuda_event for e in events])
            a.events = ctypes.cast(arr, ctypes.c_void_p)
        _check(_lib.omq_block_step(ctypes.byref(a), _ptr(self.workspace), self.workspace.numel(),
                                   _stream(stream)), "omq_block_step")
        return self.loss

    def quant_forward(self, x, dtype=torch.float32, out=None, stream=None):
        """omq_block_quant_forward: the fake-quantized block's output at the current theta
        (written into `out`, float32 or bfloat16, when given)."""
        _dev(x, out)
        y = out if out is not None else torch.empty(self.dims.M, self.dims.D, dtype=dtype,
                                                    device=self.device)
        _check(_lib.omq_block_quant_forward(ctypes.byref(self.dims), _ptr(x), _ptr(self.W["qkv"]),
                                            _ptr(self.W["o"]), _ptr(self.W["gu"]),
                                            _ptr(self.W["d"]), _ptr(self.theta), _ptr(y), _dt(y),
                                            _ptr(self.workspace), self.workspace.numel(),
                                            _stream(stream)), "omq_block_quant_forward")
        return y

    def calibrate(self, xs, y_refs, epochs, stream=None):
        """omq_block_calibrate: `epochs` passes over the samples xs [S, M, D] (BF16) with
        targets y_refs [S, M, D] (float32), one step and AdamW update per sample. Returns the
        per-step losses [epochs * S] (device tensor)."""
        _dev(xs, y_refs)
        S = xs.shape[0]
        losses = torch.empty(epochs * S, dtype=torch.float32, device=self.device)
        a = BlockCalibArgs(dims=self.dims, xs=_ptr(xs), y_refs=_ptr(y_refs), n_samples=S,
                           epochs=epochs, W_qkv=_ptr(self.W["qkv"]), W_o=_ptr(self.W["o"]),
                           W_gu=_ptr(self.W["gu"]), W_d=_ptr(self.W["d"]), theta=_ptr(self.theta),
                           d_theta=_ptr(self.d_theta), adam_m=_ptr(self.adam_m),
                           adam_v=_ptr(self.adam_v), first_step=self.t + 1, lr_lwc=self.lr_lwc,
                           lr_let=self.lr_let, losses=_ptr(losses))
        _check(_lib.omq_block_calibrate(ctypes.byref(a), _ptr(self.workspace),
                                        self.workspace.numel(), _stream(stream)),
               "omq_block_calibrate")
        self.t += epochs * S
        return losses

    def fold(self, stream=None):
        """omq_fold_pack of the four weights at the current theta (each with its linear's LET
        scale): dict name -> (packed codes, h, z)."""
        d = self.dims
        s_of = {"qkv": "s1", "o": "s_o", "gu": "s2", "d": None}
        out = {}
        for name, W in self.W.items():
            K = W.shape[1]
            G = K if d.group == 0 else d.group
            rows = W.shape[0]
            s = self.theta_part(s_of[name]) if s_of[name] else None
            gl = self.theta_part("gamma_" + name).view(rows, K // G)
            bl = self.theta_part("beta_" + name).view(rows, K // G)
            out[name] = fold_pack(W, gl, bl, d.wbits, G, s=s, stream=stream)
        return out
