"""Python binding for libzo.so, the B200 CD-RGE hot path (C ABI in include/zo.h).

Argument marshalling only: torch tensors become device pointers, the current
torch CUDA stream is passed as the cudaStream_t, and non-zero status codes
become ZOError.  Every step of the computation runs in the library's kernels;
there is no fallback.  If libzo.so is missing or fails to load, every entry
point raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libzo.so")

ZO_OK = 0
ZO_ERR_INVALID_ARG = 1
ZO_ERR_CUDA = 2
ZO_ERR_OOM = 3
ZO_ERR_UNSUPPORTED = 4
ZO_ERR_TIMEOUT = 5
ZO_ERR_NONFINITE = 6
ZO_ERR_BOUNDS = 7
ZO_ERR_NO_DEVICE = 8
ZO_DTYPE_FP32 = 0
ZO_DTYPE_BF16 = 1

# every symbol include/zo.h declares
EXPORTS = (
    "zo_create", "zo_destroy", "zo_param_layout", "zo_workspace_info", "zo_probe_losses",
    "zo_probe_losses_ex", "zo_coeffs", "zo_update", "zo_invalidate_shadow", "zo_step_host",
    "zo_sync_status", "zo_sign_words", "zo_status_string", "zo_kernel_launches",
    "zo_debug_cell_preact", "zo_profile", "zo_profile_read", "zo_probe_losses_static",
    "zo_probe_losses_slice", "zo_loss", "zo_coeffs_forward", "zo_debug_cell_stall",
    "zo_debug_cell_variant",
)
ZO_CELL_SINGLE, ZO_CELL_SINGLE_EXACT_EPS, ZO_CELL_PAIR, ZO_CELL_PAIR_EXACT_EPS, \
    ZO_CELL_PAIR_DIRECT_W, ZO_CELL_SINGLE_EPI8 = 0, 1, 2, 3, 4, 5
ZO_STATIC_SCRATCH_FLOATS = 65536
ZO_MAX_UPDATE_PROBES = 8192
ZO_KIND_CELL, ZO_KIND_LOSS, ZO_KIND_UPDATE, ZO_KIND_OTHER = 0, 1, 2, 3


class ZOError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class ModelSpec(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("vocab", "embed", "hidden", "layers", "dtype", "max_batch", "max_seq", "chunk")]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libzo.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libzo.so not found at {path}: build it with "
                          "`python -m zero_order_recurrent_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, U64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
    sig = {
        "zo_create": ([ctypes.POINTER(ModelSpec), ctypes.POINTER(P)], ctypes.c_int),
        "zo_destroy": ([P], ctypes.c_int),
        "zo_param_layout": ([P, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64),
                             ctypes.POINTER(I64), ctypes.POINTER(I32)], ctypes.c_int),
        "zo_workspace_info": ([P, ctypes.POINTER(I32), ctypes.POINTER(I64)], ctypes.c_int),
        "zo_probe_losses": ([P, P, U64, I32, F, P, P, I32, I32, P, P, P], ctypes.c_int),
        "zo_probe_losses_ex": ([P, P, U64, I32, F, P, P, I32, I32, P, P, P, P], ctypes.c_int),
        "zo_coeffs": ([P, P, P, I32, F, F, P, P], ctypes.c_int),
        "zo_update": ([P, P, U64, I32, P, P], ctypes.c_int),
        "zo_loss": ([P, P, P, P, I32, I32, P, P], ctypes.c_int),
        "zo_coeffs_forward": ([P, P, P, I32, F, F, P, P], ctypes.c_int),
        "zo_invalidate_shadow": ([P], ctypes.c_int),
        "zo_step_host": ([P, P, U64, I32, F, F, P, P, I32, I32, P, P, P], ctypes.c_int),
        "zo_sync_status": ([P, P], ctypes.c_int),
        "zo_sign_words": ([U64, I32, I64, I64, P, P], ctypes.c_int),
        "zo_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "zo_kernel_launches": ([], I64),
        "zo_debug_cell_preact": ([P, P, U64, I32, I32, F, P, I32, I32, P, P], ctypes.c_int),
        "zo_profile": ([P, I32], ctypes.c_int),
        "zo_debug_cell_stall": ([P, I32, U64, P], ctypes.c_int),
        "zo_debug_cell_variant": ([P, I32], ctypes.c_int),
        "zo_probe_losses_slice": ([P, P, U64, I32, I32, F, P, P, I32, I32, P, P, P], ctypes.c_int),
        "zo_probe_losses_static": ([ctypes.POINTER(ModelSpec), P, U64, I32, F, P, P, I32, I32, P, P,
                                    P], ctypes.c_int),
        "zo_profile_read": ([P, I32, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)],
                            ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def status_string(st: int) -> str:
    return load_library().zo_status_string(int(st)).decode()


def _check(st: int, where: str):
    if st != ZO_OK:
        raise ZOError(st, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


class Context:
    """Owns a zo_ctx (workspace and bf16 shadow on the current device)."""

    def __init__(self, vocab, embed, hidden, layers, dtype="f32", max_batch=1, max_seq=1, chunk=0):
        lib = load_library()
        self.spec = ModelSpec(vocab, embed, hidden, layers,
                              ZO_DTYPE_BF16 if dtype == "bf16" else ZO_DTYPE_FP32,
                              max_batch, max_seq, chunk)
        h = ctypes.c_void_p()
        _check(lib.zo_create(ctypes.byref(self.spec), ctypes.byref(h)), "zo_create")
        self.handle = h

    @classmethod
    def for_config(cls, cfg, max_batch=None, max_seq=None, chunk=None):
        return cls(cfg.vocab, cfg.embed, cfg.hidden, cfg.layers, cfg.dtype,
                   max_batch or cfg.batch, max_seq or cfg.seq, cfg.chunk if chunk is None else chunk)

    def close(self):
        if getattr(self, "handle", None):
            load_library().zo_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def zo_param_layout(ctx: Context):
    lib = load_library()
    d_pad, d_real = ctypes.c_int64(), ctypes.c_int64()
    n = ctypes.c_int32(32)
    off = (ctypes.c_int64 * 32)()
    num = (ctypes.c_int64 * 32)()
    _check(lib.zo_param_layout(ctx.handle, ctypes.byref(d_pad), ctypes.byref(d_real), off, num,
                               ctypes.byref(n)), "zo_param_layout")
    return d_pad.value, d_real.value, list(off[:n.value]), list(num[:n.value])


def zo_workspace_info(ctx: Context):
    lib = load_library()
    c, b = ctypes.c_int32(), ctypes.c_int64()
    _check(lib.zo_workspace_info(ctx.handle, ctypes.byref(c), ctypes.byref(b)), "zo_workspace_info")
    return c.value, b.value


def zo_probe_losses(ctx, theta, step_seed, n_pert, eps, tokens, targets, loss_plus, loss_minus,
                    row_loss=None, stream=None):
    B, T = tokens.shape
    _check(load_library().zo_probe_losses_ex(
        ctx.handle, _ptr(theta), ctypes.c_uint64(step_seed), n_pert, eps, _ptr(tokens),
        _ptr(targets), B, T, _ptr(loss_plus), _ptr(loss_minus), _ptr(row_loss), _stream(stream)),
        "zo_probe_losses")


def zo_probe_losses_slice(ctx, theta, step_seed, probe_begin, n_probes, eps, tokens, targets,
                          loss_plus, loss_minus, stream=None):
    B, T = tokens.shape
    _check(load_library().zo_probe_losses_slice(
        ctx.handle, _ptr(theta), ctypes.c_uint64(step_seed), probe_begin, n_probes, eps,
        _ptr(tokens), _ptr(targets), B, T, _ptr(loss_plus), _ptr(loss_minus), _stream(stream)),
        "zo_probe_losses_slice")


def zo_coeffs(ctx, loss_plus, loss_minus, n_pert, eps, eta, coeffs, stream=None):
    _check(load_library().zo_coeffs(ctx.handle, _ptr(loss_plus), _ptr(loss_minus), n_pert, eps,
                                    eta, _ptr(coeffs), _stream(stream)), "zo_coeffs")


def zo_loss(ctx, theta, tokens, targets, loss, stream=None):
    """L(theta) of the unperturbed forward into `loss` (one float, device)."""
    B, T = tokens.shape
    _check(load_library().zo_loss(ctx.handle, _ptr(theta), _ptr(tokens), _ptr(targets), B, T,
                                  _ptr(loss), _stream(stream)), "zo_loss")


def zo_coeffs_forward(ctx, loss_plus, loss0, n_pert, eps, eta, coeffs, stream=None):
    _check(load_library().zo_coeffs_forward(ctx.handle, _ptr(loss_plus), _ptr(loss0), n_pert, eps,
                                            eta, _ptr(coeffs), _stream(stream)),
           "zo_coeffs_forward")


def zo_update(ctx, theta, step_seed, n_pert, coeffs, stream=None):
    _check(load_library().zo_update(ctx.handle, _ptr(theta), ctypes.c_uint64(step_seed), n_pert,
                                    _ptr(coeffs), _stream(stream)), "zo_update")


def zo_invalidate_shadow(ctx):
    _check(load_library().zo_invalidate_shadow(ctx.handle), "zo_invalidate_shadow")


def zo_step_host(ctx, theta, step_seed, n_pert, eps, eta, tokens_host, targets_host,
                 loss_plus_host, loss_minus_host, stream=None):
    """tokens/targets/loss buffers: CPU tensors (ideally pinned) or numpy arrays."""
    B, T = tokens_host.shape
    _check(load_library().zo_step_host(
        ctx.handle, _ptr(theta), ctypes.c_uint64(step_seed), n_pert, eps, eta,
        _host_ptr(tokens_host), _host_ptr(targets_host), B, T, _host_ptr(loss_plus_host),
        _host_ptr(loss_minus_host), _stream(stream)), "zo_step_host")


def _host_ptr(a):
    if hasattr(a, "data_ptr"):
        return ctypes.c_void_p(a.data_ptr())
    return ctypes.c_void_p(a.ctypes.data)


def zo_sync_status(ctx, stream=None) -> int:
    return load_library().zo_sync_status(ctx.handle, _stream(stream))


def zo_sign_words(step_seed, probe, q0, n_blocks, out, stream=None):
    _check(load_library().zo_sign_words(ctypes.c_uint64(step_seed), probe, q0, n_blocks, _ptr(out),
                                        _stream(stream)), "zo_sign_words")


def zo_debug_cell_preact(ctx, theta, step_seed, probe0, n_probes, eps, tokens, preact,
                         stream=None):
    B, T = tokens.shape
    _check(load_library().zo_debug_cell_preact(
        ctx.handle, _ptr(theta), ctypes.c_uint64(step_seed), probe0, n_probes, eps, _ptr(tokens),
        B, T, _ptr(preact), _stream(stream)), "zo_debug_cell_preact")


def zo_debug_cell_stall(ctx, kind: int, wait_ns: int, stream=None):
    """Test hook: a tensor-core kernel whose waits all run out (include/zo_debug.h)."""
    _check(load_library().zo_debug_cell_stall(ctx.handle, kind, ctypes.c_uint64(wait_ns),
                                              _stream(stream)), "zo_debug_cell_stall")


def zo_debug_cell_variant(ctx, variant: int):
    """How the cell GEMMs form the perturbed operand (ZO_CELL_*, include/zo_debug.h)."""
    _check(load_library().zo_debug_cell_variant(ctx.handle, int(variant)), "zo_debug_cell_variant")


def zo_profile(ctx, enable: bool):
    _check(load_library().zo_profile(ctx.handle, 1 if enable else 0), "zo_profile")


def zo_profile_read(ctx, kind: int):
    """(launches, total_ms, total_flops, total_bytes) of one kernel kind."""
    n = ctypes.c_int64()
    ms, fl, by = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    _check(load_library().zo_profile_read(ctx.handle, kind, ctypes.byref(n), ctypes.byref(ms),
                                          ctypes.byref(fl), ctypes.byref(by)), "zo_profile_read")
    return n.value, ms.value, fl.value, by.value


def zo_probe_losses_static(spec: ModelSpec, theta, step_seed, n_pert, eps, tokens, targets,
                           loss_plus, loss_minus, stream=None) -> int:
    """Context-free fp32 probe losses that allocate no device memory (see
    include/zo.h).  Returns the status code instead of raising."""
    B, T = tokens.shape
    return load_library().zo_probe_losses_static(
        ctypes.byref(spec), _ptr(theta), ctypes.c_uint64(step_seed), n_pert, eps, _ptr(tokens),
        _ptr(targets), B, T, _ptr(loss_plus), _ptr(loss_minus), _stream(stream))


def zo_kernel_launches() -> int:
    return int(load_library().zo_kernel_launches())


def cdrge_step(ctx, theta, step_seed, n_pert, eps, eta, tokens, targets, loss_plus, loss_minus,
               coeffs, stream=None):
    """One CD-RGE update on device tensors: losses, coefficients, in-place update."""
    zo_probe_losses(ctx, theta, step_seed, n_pert, eps, tokens, targets, loss_plus, loss_minus,
                    stream=stream)
    zo_coeffs(ctx, loss_plus, loss_minus, n_pert, eps, eta, coeffs, stream=stream)
    zo_update(ctx, theta, step_seed, n_pert, coeffs, stream=stream)
