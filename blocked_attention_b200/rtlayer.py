"""ctypes binding of librtlayer.so (the C ABI declared in include/rtlayer.h).

Argument marshalling only: torch supplies device memory and streams; every
step of the layer runs in the library's CUDA kernels. There is no fallback:
if the library is missing or the device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librtlayer.so")

RT_OK, RT_ERR_INVALID_ARG, RT_ERR_UNSUPPORTED, RT_ERR_WORKSPACE, RT_ERR_CUDA, RT_ERR_TIMEOUT, RT_ERR_DEVICE = \
    0, -1, -2, -3, -4, -5, -6
RT_F32, RT_BF16 = 0, 1
RT_SCHED_BLOCKED, RT_SCHED_NAIVE = 0, 1
RT_DRIVER_GRAPH, RT_DRIVER_STREAM, RT_DRIVER_PERSISTENT = 0, 1, 2

SCHEDULES = {"blocked": RT_SCHED_BLOCKED, "naive": RT_SCHED_NAIVE}
DRIVERS = {"graph": RT_DRIVER_GRAPH, "stream": RT_DRIVER_STREAM, "persistent": RT_DRIVER_PERSISTENT}
WEIGHT_NAMES = ("W_q", "W_k", "W_v", "W_o", "W_1", "W_2")

EXPORTS = ("rt_version", "rt_status_string", "rt_last_cuda_error", "rt_cuda_error_string",
           "rt_layer_workspace_bytes", "rt_layer_forward",
           "rt_layer_sync_status", "rt_layer_host_workspace_bytes", "rt_layer_forward_host",
           "rt_embed_forward", "rt_block_fold", "rt_project_qkv", "rt_gemm_bf16",
           "rt_layer_launch_count", "rt_layer_forward_timed", "rt_project_qkv_noalloc",
           "rt_selftest_wait_timeout", "rt_layer_decode_workspace_bytes", "rt_layer_decode_step",
           "rt_project_qkv_noalloc_status", "rt_layer_recompute_workspace_bytes", "rt_layer_recompute_kv",
           "rt_layer_forward_pages", "rt_layer_backward_workspace_bytes", "rt_layer_backward",
           "rt_layer_chunked_workspace_bytes", "rt_layer_forward_chunked")

KERNEL_CLASSES = ("inv_rms", "proj", "attend", "gemm_wo", "gemm_w1", "gemm_w2", "gemm_wkv",
                  "fold_warp", "fold_tensor", "steps")
RT_KC_FOLD_LEVEL0 = 16
RT_KC_COUNT = 32

_lib = None


class RTError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn} failed: {status} ({status_string(status)})"
        self.cuda_error = 0
        if status == RT_ERR_CUDA:
            self.cuda_error = int(lib().rt_last_cuda_error())
            msg += f": CUDA error {self.cuda_error} ({lib().rt_cuda_error_string(self.cuda_error).decode()})"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """Load librtlayer.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m blocked_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    fp = ctypes.POINTER(ctypes.c_float)
    L.rt_version.restype = i
    L.rt_status_string.restype = ctypes.c_char_p
    L.rt_status_string.argtypes = [i]
    L.rt_last_cuda_error.restype = i
    L.rt_last_cuda_error.argtypes = []
    L.rt_cuda_error_string.restype = ctypes.c_char_p
    L.rt_cuda_error_string.argtypes = [i]
    L.rt_layer_workspace_bytes.restype = sz
    L.rt_layer_workspace_bytes.argtypes = [i] * 7
    L.rt_layer_host_workspace_bytes.restype = sz
    L.rt_layer_host_workspace_bytes.argtypes = [i] * 7
    fwd_args = [vp] * 7 + [i] * 8 + [vp] * 4 + [sz, vp]
    L.rt_layer_forward.restype = i
    L.rt_layer_forward.argtypes = fwd_args
    L.rt_layer_forward_host.restype = i
    L.rt_layer_forward_host.argtypes = fwd_args
    L.rt_layer_backward_workspace_bytes.restype = sz
    L.rt_layer_backward_workspace_bytes.argtypes = [i] * 6
    L.rt_layer_backward.restype = i
    L.rt_layer_backward.argtypes = [vp] * 13 + [i] * 6 + [vp] * 8 + [sz, vp]
    L.rt_layer_chunked_workspace_bytes.restype = sz
    L.rt_layer_chunked_workspace_bytes.argtypes = [i] * 6
    L.rt_layer_forward_chunked.restype = i
    L.rt_layer_forward_chunked.argtypes = [vp] * 7 + [i] * 6 + [vp] * 4 + [sz, vp]
    L.rt_layer_forward_pages.restype = i
    L.rt_layer_forward_pages.argtypes = [vp] * 7 + [i] * 6 + [vp] * 4 + [sz, vp, i]
    L.rt_layer_sync_status.restype = i
    L.rt_layer_sync_status.argtypes = [vp, vp]
    L.rt_embed_forward.restype = i
    L.rt_embed_forward.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp]
    L.rt_block_fold.restype = i
    L.rt_block_fold.argtypes = [vp, i, vp, vp, i, fp, fp, fp] + [i] * 7 + [i, vp, vp]
    L.rt_project_qkv.restype = i
    L.rt_project_qkv.argtypes = [vp, vp, i, i, i, i, vp, vp, vp, vp]
    L.rt_gemm_bf16.restype = i
    L.rt_gemm_bf16.argtypes = [vp, vp, fp, i, i, i, vp, vp]
    L.rt_layer_launch_count.restype = ctypes.c_long
    L.rt_layer_launch_count.argtypes = [i] * 8
    L.rt_layer_forward_timed.restype = i
    L.rt_layer_forward_timed.argtypes = [vp] * 7 + [i] * 7 + [vp] * 4 + [sz, vp, fp,
                                                                         ctypes.POINTER(ctypes.c_int), i]
    L.rt_project_qkv_noalloc.restype = i
    L.rt_project_qkv_noalloc.argtypes = [vp, vp, i, i, i, vp, vp]
    L.rt_project_qkv_noalloc_status.restype = i
    L.rt_project_qkv_noalloc_status.argtypes = [vp]
    L.rt_layer_recompute_workspace_bytes.restype = sz
    L.rt_layer_recompute_workspace_bytes.argtypes = [i] * 3
    L.rt_layer_recompute_kv.restype = i
    L.rt_layer_recompute_kv.argtypes = [vp] * 3 + [i] * 3 + [vp] * 3 + [sz, vp]
    L.rt_selftest_wait_timeout.restype = i
    L.rt_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp, vp]
    L.rt_layer_decode_workspace_bytes.restype = sz
    L.rt_layer_decode_workspace_bytes.argtypes = [i] * 4
    L.rt_layer_decode_step.restype = i
    L.rt_layer_decode_step.argtypes = [vp] * 7 + [i] * 6 + [vp] * 4 + [sz, vp]
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().rt_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != RT_OK:
        raise RTError(fn, status)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return RT_F32
    if t == torch.bfloat16:
        return RT_BF16
    raise ValueError(f"unsupported dtype {t}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _fptr(t):
    return ctypes.cast(ctypes.c_void_p(t.data_ptr()), ctypes.POINTER(ctypes.c_float))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------
def workspace_bytes(B, N, d, H, d_ff, dtype=torch.bfloat16, schedule="blocked") -> int:
    return int(lib().rt_layer_workspace_bytes(B, N, d, H, d_ff, _dtype_code(dtype), SCHEDULES[schedule]))


def host_workspace_bytes(B, N, d, H, d_ff, dtype=torch.bfloat16, schedule="blocked") -> int:
    return int(lib().rt_layer_host_workspace_bytes(B, N, d, H, d_ff, _dtype_code(dtype), SCHEDULES[schedule]))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    # torch's caching allocator returns blocks aligned to at least 512 bytes
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def layer_forward(x: torch.Tensor, W: dict, H: int, d_ff: int | None = None, schedule: str = "blocked",
                  driver: str = "graph", out=None, workspace: torch.Tensor | None = None, stream=None):
    """rt_layer_forward on device tensors. x: [B, N, d] (fp32 or bf16, cuda);
    W: dict of W_q, W_k, W_v, W_o [d, d], W_1 [d_ff, d], W_2 [d, d_ff].
    Returns (z [B, N, d], K [N, B, d], V [N, B, d]) -- K, V position-major."""
    B, N, d = x.shape
    d_ff = d_ff or W["W_1"].shape[0]
    code = _dtype_code(x.dtype)
    for n in WEIGHT_NAMES:
        if W[n].dtype != x.dtype or not W[n].is_contiguous() or W[n].device != x.device:
            raise ValueError(f"weight {n} must be a contiguous {x.dtype} tensor on {x.device}")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if out is None:
        z = torch.empty_like(x)
        K = torch.empty((N, B, d), dtype=x.dtype, device=x.device)
        V = torch.empty_like(K)
    else:
        z, K, V = out
    nbytes = workspace_bytes(B, N, d, H, d_ff, x.dtype, schedule)
    if nbytes == 0:
        raise RTError("rt_layer_workspace_bytes", RT_ERR_UNSUPPORTED)
    if workspace is None:
        workspace = alloc_workspace(nbytes, x.device)
    rc = lib().rt_layer_forward(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, N, d, H, d_ff, code,
                                SCHEDULES[schedule], DRIVERS[driver], _ptr(z), _ptr(K), _ptr(V),
                                _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("rt_layer_forward", rc)
    return z, K, V


def layer_forward_pages(x: torch.Tensor, W: dict, H: int, L: int = 1, out=None,
                        workspace: torch.Tensor | None = None, stream=None, driver: str = "graph"):
    """rt_layer_forward_pages: the layer in the paper's own parameterisation
    (per-head unit-RMS queries and keys, no softmax scale, RMS without eps,
    branches scaled by 1/sqrt(L)); bf16 device tensors as in layer_forward."""
    B, N, d = x.shape
    d_ff = W["W_1"].shape[0]
    for n in WEIGHT_NAMES:
        if W[n].dtype != torch.bfloat16 or not W[n].is_contiguous() or W[n].device != x.device:
            raise ValueError(f"weight {n} must be a contiguous bf16 tensor on {x.device}")
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 tensor")
    if out is None:
        z = torch.empty_like(x)
        K = torch.empty((N, B, d), dtype=x.dtype, device=x.device)
        V = torch.empty_like(K)
    else:
        z, K, V = out
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(B, N, d, H, d_ff), x.device)
    rc = lib().rt_layer_forward_pages(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, N, d, H, d_ff, L,
                                      _ptr(z), _ptr(K), _ptr(V), _ptr(workspace),
                                      ctypes.c_size_t(workspace.numel()), _stream(stream), DRIVERS[driver])
    _check("rt_layer_forward_pages", rc)
    return z, K, V


def layer_backward(x: torch.Tensor, W: dict, H: int, z: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                   dz: torch.Tensor, dK: torch.Tensor, dV: torch.Tensor, workspace: torch.Tensor | None = None,
                   stream=None):
    """rt_layer_backward: gradients of sum(z*dz) + sum(K*dK) + sum(V*dV) for
    x [B, N, d], the weights W, the forward's outputs z [B, N, d] and K, V
    [N, B, d] (position-major), and upstream dz, dK, dV of the same shapes;
    all fp32 or all bf16 (fp32 arithmetic either way). Returns
    (dx, {name: dW})."""
    B, N, d = x.shape
    d_ff = W["W_1"].shape[0]
    code = _dtype_code(x.dtype)
    tensors = (x, z, K, V, dz, dK, dV, *[W[n] for n in WEIGHT_NAMES])
    for tsr in tensors:
        if tsr.dtype != x.dtype or not tsr.is_contiguous() or tsr.device != x.device:
            raise ValueError("backward tensors must be contiguous tensors of one dtype on one device")
    dx = torch.empty_like(x)
    dW = {n: torch.empty_like(W[n]) for n in WEIGHT_NAMES}
    nbytes = int(lib().rt_layer_backward_workspace_bytes(B, N, d, H, d_ff, code))
    if nbytes == 0:
        raise RTError("rt_layer_backward_workspace_bytes", RT_ERR_UNSUPPORTED)
    if workspace is None:
        workspace = alloc_workspace(nbytes, x.device)
    rc = lib().rt_layer_backward(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], _ptr(z), _ptr(K), _ptr(V),
                                 _ptr(dz), _ptr(dK), _ptr(dV), B, N, d, H, d_ff, code, _ptr(dx),
                                 *[_ptr(dW[n]) for n in WEIGHT_NAMES], _ptr(workspace),
                                 ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("rt_layer_backward", rc)
    return dx, dW


def layer_forward_chunked(x: torch.Tensor, W: dict, H: int, C: int, out=None,
                          workspace: torch.Tensor | None = None, stream=None):
    """rt_layer_forward_chunked: the block-wise recurrence with chunks of C
    positions; bf16 device tensors as in layer_forward."""
    B, N, d = x.shape
    d_ff = W["W_1"].shape[0]
    for n in WEIGHT_NAMES:
        if W[n].dtype != torch.bfloat16 or not W[n].is_contiguous() or W[n].device != x.device:
            raise ValueError(f"weight {n} must be a contiguous bf16 tensor on {x.device}")
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 tensor")
    if out is None:
        z = torch.empty_like(x)
        K = torch.empty((N, B, d), dtype=x.dtype, device=x.device)
        V = torch.empty_like(K)
    else:
        z, K, V = out
    if workspace is None:
        nbytes = int(lib().rt_layer_chunked_workspace_bytes(B, N, d, H, d_ff, C))
        if nbytes == 0:
            raise RTError("rt_layer_chunked_workspace_bytes", RT_ERR_UNSUPPORTED)
        workspace = alloc_workspace(nbytes, x.device)
    rc = lib().rt_layer_forward_chunked(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, N, d, H, d_ff, C,
                                        _ptr(z), _ptr(K), _ptr(V), _ptr(workspace),
                                        ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("rt_layer_forward_chunked", rc)
    return z, K, V


def launch_count(B, N, d, H, d_ff, dtype=torch.bfloat16, schedule="blocked", driver="graph") -> int:
    return int(lib().rt_layer_launch_count(B, N, d, H, d_ff, _dtype_code(dtype), SCHEDULES[schedule],
                                           DRIVERS[driver]))


def layer_forward_timed(x: torch.Tensor, W: dict, H: int, out, workspace: torch.Tensor,
                        d_ff: int | None = None, schedule: str = "blocked", stream=None) -> dict:
    """rt_layer_forward_timed: one forward with CUDA events around every
    kernel; returns {class: (total_ms, launches)} (synchronises the stream)."""
    B, N, d = x.shape
    d_ff = d_ff or W["W_1"].shape[0]
    z, K, V = out
    ms = (ctypes.c_float * RT_KC_COUNT)()
    cnt = (ctypes.c_int * RT_KC_COUNT)()
    rc = lib().rt_layer_forward_timed(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, N, d, H, d_ff,
                                      _dtype_code(x.dtype), SCHEDULES[schedule], _ptr(z), _ptr(K), _ptr(V),
                                      _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream),
                                      ms, cnt, RT_KC_COUNT)
    _check("rt_layer_forward_timed", rc)
    out = {name: (float(ms[i]), int(cnt[i])) for i, name in enumerate(KERNEL_CLASSES) if cnt[i] > 0}
    for lv in range(RT_KC_COUNT - RT_KC_FOLD_LEVEL0):
        c = RT_KC_FOLD_LEVEL0 + lv
        if cnt[c] > 0:
            out[f"fold_lb{1 << lv}"] = (float(ms[c]), int(cnt[c]))
    return out


def selftest_wait_timeout(limit_ns: int, workspace: torch.Tensor, stream=None):
    """Enqueue the bounded-wait self-test (see rt_selftest_wait_timeout)."""
    _check("rt_selftest_wait_timeout", lib().rt_selftest_wait_timeout(int(limit_ns), _ptr(workspace), _stream(stream)))


def decode_workspace_bytes(B: int, d: int, H: int, d_ff: int) -> int:
    return int(lib().rt_layer_decode_workspace_bytes(B, d, H, d_ff))


def layer_decode_step(x_t: torch.Tensor, W: dict, H: int, t: int, K_cache: torch.Tensor, V_cache: torch.Tensor,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """rt_layer_decode_step: x_t [B, d] bf16 on cuda; K_cache, V_cache
    [capacity, B, d] bf16 holding positions 1..t-1 in rows 0..t-2. Writes the
    new persistent pair to row t-1 of the caches and returns z_t [B, d]."""
    B, d = x_t.shape
    d_ff = W["W_1"].shape[0]
    cap = K_cache.shape[0]
    for tsr in (x_t, K_cache, V_cache, *[W[n] for n in WEIGHT_NAMES]):
        if tsr.dtype != torch.bfloat16 or not tsr.is_contiguous() or tsr.device != x_t.device:
            raise ValueError("decode step tensors must be contiguous bf16 tensors on one device")
    if tuple(K_cache.shape) != (cap, B, d) or tuple(V_cache.shape) != (cap, B, d):
        raise ValueError("K_cache, V_cache must be [capacity, B, d]")
    z = out if out is not None else torch.empty_like(x_t)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_bytes(B, d, H, d_ff), x_t.device)
    rc = lib().rt_layer_decode_step(_ptr(x_t), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, t, cap, d, H, d_ff,
                                    _ptr(z), _ptr(K_cache), _ptr(V_cache), _ptr(workspace),
                                    ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("rt_layer_decode_step", rc)
    return z


def recompute_kv(z: torch.Tensor, W_k: torch.Tensor, W_v: torch.Tensor, out=None,
                 workspace: torch.Tensor | None = None, stream=None):
    """rt_layer_recompute_kv: the persistent pairs of every position rebuilt
    from stored outputs z [B, N, d] (bf16, cuda). Returns (K, V), each
    position-major [N, B, d]."""
    B, N, d = z.shape
    for tsr in (z, W_k, W_v):
        if tsr.dtype != torch.bfloat16 or not tsr.is_contiguous() or tsr.device != z.device:
            raise ValueError("recompute tensors must be contiguous bf16 tensors on one device")
    if out is None:
        K = torch.empty((N, B, d), dtype=z.dtype, device=z.device)
        V = torch.empty_like(K)
    else:
        K, V = out
    nbytes = int(lib().rt_layer_recompute_workspace_bytes(B, N, d))
    if nbytes == 0:
        raise RTError("rt_layer_recompute_workspace_bytes", RT_ERR_UNSUPPORTED)
    if workspace is None:
        workspace = alloc_workspace(nbytes, z.device)
    rc = lib().rt_layer_recompute_kv(_ptr(z), _ptr(W_k), _ptr(W_v), B, N, d, _ptr(K), _ptr(V), _ptr(workspace),
                                     ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("rt_layer_recompute_kv", rc)
    return K, V


def sync_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().rt_layer_sync_status(_ptr(workspace), _stream(stream)))


def layer_forward_host(x: torch.Tensor, W: dict, H: int, out, workspace: torch.Tensor, d_ff: int | None = None,
                       schedule: str = "blocked", driver: str = "graph", stream=None):
    """rt_layer_forward_host: x, W and out=(z, K, V) are HOST tensors (pinned
    for asynchronous copies); workspace is a device buffer of
    host_workspace_bytes(...) bytes. Returns once enqueued."""
    B, N, d = x.shape
    d_ff = d_ff or W["W_1"].shape[0]
    z, K, V = out
    rc = lib().rt_layer_forward_host(_ptr(x), *[_ptr(W[n]) for n in WEIGHT_NAMES], B, N, d, H, d_ff,
                                     _dtype_code(x.dtype), SCHEDULES[schedule], DRIVERS[driver], _ptr(z),
                                     _ptr(K), _ptr(V), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                     _stream(stream))
    _check("rt_layer_forward_host", rc)


# --------------------------------------------------------------------------
# stack front end and component entry points
# --------------------------------------------------------------------------
def embed_forward(ids: torch.Tensor, E: torch.Tensor, workspace: torch.Tensor | None = None, stream=None):
    B, N = ids.shape
    vocab, d = E.shape
    x = torch.empty((B, N, d), dtype=E.dtype, device=E.device)
    rc = lib().rt_embed_forward(_ptr(ids), _ptr(E), B, N, vocab, d, _dtype_code(E.dtype), _ptr(x),
                                _ptr(workspace), _stream(stream))
    _check("rt_embed_forward", rc)
    return x


def _err_word(err, device):
    """The caller's device error word, or a fresh zeroed one (owned here)."""
    if err is not None:
        return err, False
    return torch.zeros(256, dtype=torch.uint8, device=device), True


def _finish(fn: str, err, owned: bool, stream):
    """When the binding owns the error word, read it (synchronises the stream)
    and raise on a device-side error; otherwise the caller reads it with
    sync_status(err)."""
    if owned:
        _check(fn, sync_status(err, stream))


def block_fold(Q, K, V, m, l, o, H: int, d_h: int, q0: int, nq: int, k0: int, nk: int, err=None, stream=None):
    """rt_block_fold: Q [n_pos, B, q_stride], K/V [n_pos, B, kv_stride];
    m, l [n_pos, B, H] and o [n_pos, B, H*d_h] fp32 updated in place.
    err: device error word (None: a private one, checked before returning)."""
    B = Q.shape[1]
    err, owned = _err_word(err, Q.device)
    rc = lib().rt_block_fold(_ptr(Q), Q.shape[2], _ptr(K), _ptr(V), K.shape[2], _fptr(m), _fptr(l), _fptr(o),
                             B, H, d_h, q0, nq, k0, nk, _dtype_code(Q.dtype), _ptr(err), _stream(stream))
    _check("rt_block_fold", rc)
    _finish("rt_block_fold", err, owned, stream)


def project_qkv(x: torch.Tensor, W_qkv: torch.Tensor, err=None, stream=None):
    """rt_project_qkv: x [B, N, d] -> QKV position-major [N, B, 3d].
    err: device error word (None: a private one, checked before returning)."""
    B, N, d = x.shape
    qkv = torch.empty((N, B, 3 * d), dtype=x.dtype, device=x.device)
    scratch = torch.empty(B * N * (1 if x.dtype == torch.bfloat16 else d), dtype=torch.float32, device=x.device)
    err, owned = _err_word(err, x.device)
    rc = lib().rt_project_qkv(_ptr(x), _ptr(W_qkv), B, N, d, _dtype_code(x.dtype), _ptr(qkv), _ptr(scratch),
                              _ptr(err), _stream(stream))
    _check("rt_project_qkv", rc)
    _finish("rt_project_qkv", err, owned, stream)
    return qkv


def project_qkv_noalloc(x: torch.Tensor, W_qkv: torch.Tensor, out: torch.Tensor, stream=None):
    """rt_project_qkv_noalloc: bf16 projection into the caller's `out`
    ([N, B, 3d]) with the library's fixed scratch array (B*N <= 1048576)."""
    B, N, d = x.shape
    rc = lib().rt_project_qkv_noalloc(_ptr(x), _ptr(W_qkv), B, N, d, _ptr(out), _stream(stream))
    _check("rt_project_qkv_noalloc", rc)
    return out


def project_qkv_noalloc_status(stream=None) -> int:
    """rt_project_qkv_noalloc_status: synchronises the stream, then reads and
    clears the library's error word of the allocation-free projection."""
    return int(lib().rt_project_qkv_noalloc_status(_stream(stream)))


def gemm_bf16(A: torch.Tensor, W: torch.Tensor, err=None, stream=None):
    """rt_gemm_bf16: C = A W^T (bf16 operands, fp32 C).
    err: device error word (None: a private one, checked before returning)."""
    M, Kd = A.shape
    Nout = W.shape[0]
    C = torch.empty((M, Nout), dtype=torch.float32, device=A.device)
    err, owned = _err_word(err, A.device)
    rc = lib().rt_gemm_bf16(_ptr(A), _ptr(W), _fptr(C), M, Nout, Kd, _ptr(err), _stream(stream))
    _check("rt_gemm_bf16", rc)
    _finish("rt_gemm_bf16", err, owned, stream)
    return C
