"""Python binding of libkimodo.so, the B200 two-stage DDIM denoiser.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if the shared library is missing or cannot
be loaded, every entry point raises.  Tensors may be torch tensors (CUDA or CPU)
or numpy arrays; the library detects host versus device memory itself.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = ["KimodoError", "load_library", "Kimodo", "N_PARAMS", "FP32", "BF16", "NET_ROOT", "NET_BODY"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkimodo.so")

N_PARAMS = 281_963_799
FP32, BF16 = 0, 1
NET_ROOT, NET_BODY = 0, 1
TEXT_DIM, MOTION_DIM, ROOT_DIM, BODY_DIM = 4096, 279, 5, 274
STATUS = {0: "OK", -1: "EINVAL", -2: "ENOMEM", -3: "ECUDA", -4: "EUNSUPPORTED", -5: "ETIMEOUT"}

# (name, restype, argtypes) for every symbol declared in include/kimodo.h
_P, _I, _F, _SZ, _LL, _D = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong, ctypes.c_void_p
SIGNATURES = [
    ("kimodo_load_weights", _I, [ctypes.POINTER(_P), _P, _SZ, _I, _I]),
    ("kimodo_denoiser_forward", _I, [_P, _I, _P, _P, _I, _P, _I, _I, _P, _P]),
    ("kimodo_denoiser_forward_noalloc", _I, [_P, _I, _P, _P, _I, _P, _I, _I, _P, _P]),
    ("kimodo_ddim_step", _I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P]),
    ("kimodo_ddim_sample", _I, [_P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P, _P]),
    ("kimodo_ddim_step_ex", _I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _P]),
    ("kimodo_ddim_sample_ex", _I, [_P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P, _P, _P]),
    ("kimodo_sync_status", _I, [_P, _P]),
    ("kimodo_wait_selftest", _I, [_P, _I, _P]),
    ("kimodo_profile_enable", _I, [_P, _I]),
    ("kimodo_profile_read", _I, [_P, _I, _P, _P, _P, _P]),
    ("kimodo_last_launch_count", _LL, [_P]),
    ("kimodo_free", None, [_P]),
    ("kimodo_last_error", ctypes.c_char_p, []),
    # include/kimodo_kernels.h
    ("kimodo_gemm_bf16", _I, [_P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    ("kimodo_gemm_bf16_pair", _I, [_P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    ("kimodo_gemm_f32", _I, [_P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I, _P]),
    ("kimodo_attention_bf16", _I, [_P, _P, _P, _I, _I, _P]),
    ("kimodo_attention_f32", _I, [_P, _P, _P, _I, _I, _P]),
    ("kimodo_layernorm", _I, [_P, _P, _I, _P, _P, _I, _P]),
    ("kimodo_global_to_local_root", _I, [_P, _P, _P, _I, _I, _P, _P]),
]
EPI_BIAS, EPI_BIAS_GELU, EPI_BIAS_SILU, EPI_BIAS_RESID = 0, 1, 2, 3


SCHEDULES = {"linear": 0, "cosine": 1}


class SamplerOptions(ctypes.Structure):
    """struct kimodo_sampler of include/kimodo.h."""
    _fields_ = [("schedule", ctypes.c_int), ("eta", ctypes.c_float), ("step_noise", ctypes.c_void_p),
                ("text_batch", ctypes.c_int)]


class KimodoError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"kimodo {STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libkimodo.so and declare its C signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m transformer_denoiser_b200.build`")
    lib = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        raise KimodoError(status, _lib.kimodo_last_error().decode())


def _ptr(a):
    """Data pointer of a contiguous torch tensor or numpy array."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        if not a.flags.c_contiguous:
            raise ValueError("numpy arrays must be C-contiguous")
        return a.ctypes.data
    if not a.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return a.data_ptr()


def _ptr_rows(a):
    """Data pointer of a row-major 2-D tensor whose rows may be padded (stride(1) == 1)."""
    if a is None:
        return None
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("need a 2-D tensor with unit column stride")
    return a.data_ptr()


def _is_cuda(a):
    return hasattr(a, "is_cuda") and a.is_cuda


def _stream(stream, *tensors):
    if stream is not None:
        return stream
    if any(_is_cuda(t) for t in tensors):
        import torch
        return torch.cuda.current_stream().cuda_stream
    return None


def _like(ref, shape, dtype_np=np.float32):
    if _is_cuda(ref):
        import torch
        return torch.empty(shape, dtype=torch.float32, device=ref.device)
    return np.empty(shape, dtype=dtype_np)


def _f32(a):
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a, dtype=np.float32)
    return a.contiguous()


def _i32(a):
    if isinstance(a, np.ndarray) or isinstance(a, (list, tuple)):
        return np.ascontiguousarray(np.asarray(a), dtype=np.int32)
    return a.contiguous()


def _cur_stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------ kernel-level calls (torch CUDA tensors)

def gemm_bf16(A, W, bias, epilogue=EPI_BIAS, out_f32=False, resid=None, out=None, K=None, tile_n=0, pair=False):
    """out = epilogue(A[:, :K] W[:, :K]^T + bias) on the tcgen05 GEMM (A, W bf16 CUDA tensors);
    pair=True runs the CTA-pair kernel (256-row tiles)."""
    import torch
    lib = load_library()
    M, N = A.shape[0], W.shape[0]
    K = A.shape[1] if K is None else K
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if out_f32 else torch.bfloat16, device=A.device)
    args = [_ptr_rows(A), A.stride(0), _ptr_rows(W), W.stride(0), _ptr(bias), _ptr_rows(resid),
            0 if resid is None else resid.stride(0), _ptr_rows(out), out.stride(0), M, N, K,
            int(epilogue), int(bool(out_f32))]
    fn = lib.kimodo_gemm_bf16_pair if pair else lib.kimodo_gemm_bf16
    _check(fn(*args, int(tile_n), _cur_stream()))
    return out


def gemm_f32(A, W, bias, epilogue=EPI_BIAS, resid=None, out=None, K=None):
    import torch
    lib = load_library()
    M, N = A.shape[0], W.shape[0]
    K = A.shape[1] if K is None else K
    out = torch.empty((M, N), dtype=torch.float32, device=A.device) if out is None else out
    _check(lib.kimodo_gemm_f32(_ptr(A), A.stride(0), _ptr(W), W.stride(0), _ptr(bias), _ptr(resid),
                               0 if resid is None else resid.stride(0), _ptr(out), out.stride(0), M, N, K,
                               int(epilogue), _cur_stream()))
    return out


def attention(qkv, lengths, nseq, S):
    """Masked attention over qkv [nseq*S, 3072] (CUDA tensor): bf16 runs the tcgen05
    kernel, fp32 the fp32 one."""
    import torch
    lib = load_library()
    out = torch.empty((nseq * S, 1024), dtype=qkv.dtype, device=qkv.device)
    fn = lib.kimodo_attention_bf16 if qkv.dtype == torch.bfloat16 else lib.kimodo_attention_f32
    _check(fn(_ptr(qkv), _ptr(out), _ptr(lengths), nseq, S, _cur_stream()))
    return out


def layernorm(y, gamma, beta, out_bf16=True):
    import torch
    lib = load_library()
    out = torch.empty(y.shape, dtype=torch.bfloat16 if out_bf16 else torch.float32, device=y.device)
    _check(lib.kimodo_layernorm(_ptr(y), _ptr(out), int(bool(out_bf16)), _ptr(gamma), _ptr(beta), y.shape[0],
                                _cur_stream()))
    return out


def global_to_local_root(root, x, lengths):
    """[x[..., 5:] | globalRootToLocalRoot(root)] (fp32 CUDA tensors root [B, T, 5],
    x [B, T, 279], int32 lengths [B])."""
    import torch
    lib = load_library()
    B, T = x.shape[0], x.shape[1]
    out = torch.empty((B, T, MOTION_DIM), dtype=torch.float32, device=x.device)
    _check(lib.kimodo_global_to_local_root(_ptr(root), _ptr(x), _ptr(lengths), B, T, _ptr(out), _cur_stream()))
    return out


class Kimodo:
    """A loaded denoiser pair on one GPU (wraps a kimodo_ctx)."""

    def __init__(self, blob, precision: int = BF16, device: int = 0):
        lib = load_library()
        self._lib = lib
        self._ctx = ctypes.c_void_p()
        blob = _f32(blob)
        n = int(blob.size if isinstance(blob, np.ndarray) else blob.numel())
        _check(lib.kimodo_load_weights(ctypes.byref(self._ctx), _ptr(blob), n, int(precision), int(device)))
        self.precision = precision
        self.device = device

    def close(self):
        if getattr(self, "_ctx", None) and self._ctx.value:
            self._lib.kimodo_free(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---------------------------------------------------------------- entry points
    def denoiser_forward(self, net, x, emb, t, lengths, out=None, stream=None):
        x, emb, lengths = _f32(x), _f32(emb), _i32(lengths)
        B, T = x.shape[0], x.shape[1]
        dout = ROOT_DIM if net == NET_ROOT else BODY_DIM
        out = _like(x, (B, T, dout)) if out is None else out
        _check(self._lib.kimodo_denoiser_forward(self._ctx, int(net), _ptr(x), _ptr(emb), int(t), _ptr(lengths),
                                                 B, T, _ptr(out), _stream(stream, x, out)))
        return out

    def denoiser_forward_noalloc(self, net, x, emb, t, lengths, out=None, stream=None):
        """kimodo_denoiser_forward_noalloc: same result, no device allocation (size limits apply)."""
        x, emb, lengths = _f32(x), _f32(emb), _i32(lengths)
        B, T = x.shape[0], x.shape[1]
        dout = ROOT_DIM if net == NET_ROOT else BODY_DIM
        out = _like(x, (B, T, dout)) if out is None else out
        _check(self._lib.kimodo_denoiser_forward_noalloc(self._ctx, int(net), _ptr(x), _ptr(emb), int(t),
                                                         _ptr(lengths), B, T, _ptr(out), _stream(stream, x, out)))
        return out

    @staticmethod
    def _options(schedule, eta, step_noise, text_batch=0):
        """kimodo_sampler for the _ex calls, or None for the defaults (linear, eta 0, one
        text row per sequence)."""
        if schedule == "linear" and float(eta) == 0.0 and not text_batch:
            return None, None
        z = None if step_noise is None else _f32(step_noise)
        return SamplerOptions(SCHEDULES[schedule], float(eta), _ptr(z), int(text_batch)), z

    def ddim_step(self, x_t, text_emb, null_emb, lengths, t, t_prev, cfg_scale, out=None, stream=None,
                  schedule="linear", eta=0.0, step_noise=None):
        x_t, text_emb, null_emb, lengths = _f32(x_t), _f32(text_emb), _f32(null_emb), _i32(lengths)
        B, T = x_t.shape[0], x_t.shape[1]
        nb = 1 if null_emb.ndim == 1 else null_emb.shape[0]
        out = _like(x_t, (B, T, MOTION_DIM)) if out is None else out
        opts, z = self._options(schedule, eta, step_noise, text_emb.shape[0] if text_emb.shape[0] != B else 0)
        if opts is None:
            _check(self._lib.kimodo_ddim_step(self._ctx, _ptr(x_t), _ptr(text_emb), _ptr(null_emb), nb,
                                              _ptr(lengths), B, T, int(t), int(t_prev), float(cfg_scale), _ptr(out),
                                              _stream(stream, x_t, out)))
        else:
            _check(self._lib.kimodo_ddim_step_ex(self._ctx, _ptr(x_t), _ptr(text_emb), _ptr(null_emb), nb,
                                                 _ptr(lengths), B, T, int(t), int(t_prev), float(cfg_scale),
                                                 ctypes.byref(opts), _ptr(out), _stream(stream, x_t, out)))
        return out

    def ddim_sample(self, text_emb, null_emb, noise, lengths, steps, cfg_scale, out=None, stream=None,
                    schedule="linear", eta=0.0, step_noise=None):
        """Full sampler; schedule "linear" or "cosine", eta in [0, 1] with step_noise
        [steps, B, T, 279] standard-normal draws when eta > 0.  text_emb may have fewer
        rows than the batch (a divisor of B): variations, row b // (B // rows) per sequence."""
        text_emb, null_emb, noise, lengths = _f32(text_emb), _f32(null_emb), _f32(noise), _i32(lengths)
        B, T = noise.shape[0], noise.shape[1]
        nb = 1 if null_emb.ndim == 1 else null_emb.shape[0]
        out = _like(noise, (B, T, MOTION_DIM)) if out is None else out
        opts, z = self._options(schedule, eta, step_noise, text_emb.shape[0] if text_emb.shape[0] != B else 0)
        if opts is None:
            _check(self._lib.kimodo_ddim_sample(self._ctx, _ptr(text_emb), _ptr(null_emb), nb, _ptr(noise),
                                                _ptr(lengths), B, T, int(steps), float(cfg_scale), _ptr(out),
                                                _stream(stream, noise, out)))
        else:
            _check(self._lib.kimodo_ddim_sample_ex(self._ctx, _ptr(text_emb), _ptr(null_emb), nb, _ptr(noise),
                                                   _ptr(lengths), B, T, int(steps), float(cfg_scale),
                                                   ctypes.byref(opts), _ptr(out), _stream(stream, noise, out)))
        return out

    def wait_selftest(self, limit_us: int, stream=None):
        """kimodo_wait_selftest: a kernel whose bounded wait runs out and records a timeout."""
        _check(self._lib.kimodo_wait_selftest(self._ctx, int(limit_us), stream))

    def sync_status(self, stream=None):
        _check(self._lib.kimodo_sync_status(self._ctx, stream))

    def profile_enable(self, on: bool = True):
        _check(self._lib.kimodo_profile_enable(self._ctx, int(bool(on))))

    def profile_read(self, n_classes: int = 6):
        ms = (ctypes.c_double * n_classes)()
        cnt = (ctypes.c_longlong * n_classes)()
        fl = (ctypes.c_double * n_classes)()
        by = (ctypes.c_double * n_classes)()
        _check(self._lib.kimodo_profile_read(self._ctx, n_classes, ms, cnt, fl, by))
        names = ["gemm_tc", "attention", "layernorm", "motion", "gemm_f32", "setup", "c6", "c7"]
        return {names[i]: dict(ms=ms[i], launches=cnt[i], flops=fl[i], bytes=by[i]) for i in range(n_classes)}

    def last_launch_count(self) -> int:
        return int(self._lib.kimodo_last_launch_count(self._ctx))
