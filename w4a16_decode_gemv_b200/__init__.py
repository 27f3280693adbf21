"""Python binding of the w4a16 C ABI (include/w4a16.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libw4a16.so``.  PyTorch supplies device memory and the current
stream.  There is no CPU fallback: if the library is missing or the tensors
are not on a CUDA device, the call raises.

Packed weights are uint32 bit patterns kept in ``torch.int32`` tensors.
"""
from __future__ import annotations

import ctypes
import os

import torch

ASYM = 0
SYM = 1
GROUP = 128
LAYOUT_VERSION = 1

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4a16.so")
_lib = None
_workspaces: dict = {}


class W4A16Error(RuntimeError):
    pass


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libw4a16.so once and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise W4A16Error(f"{_LIB_PATH} is missing: build it with `python -m w4a16_decode_gemv_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i, d, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
    lib.awq_act_scale.argtypes = [vp, i, i, d, vp, vp]
    lib.awq_act_scale.restype = i
    lib.awq_quantize_pack.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, vp]
    lib.awq_quantize_pack.restype = i
    lib.w4a16_gemm_workspace_size.argtypes = [i, i, i, i]
    lib.w4a16_gemm_workspace_size.restype = sz
    lib.w4a16_gemm.argtypes = [vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp]
    lib.w4a16_gemm.restype = i
    lib.w4a16_gemv_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, vp, vp]
    lib.w4a16_gemv_noalloc.restype = i
    lib.w4a16_gemv_noalloc_max_scratch.argtypes = []
    lib.w4a16_gemv_noalloc_max_scratch.restype = sz
    lib.w4a16_gemv_noalloc_check.argtypes = [vp]
    lib.w4a16_gemv_noalloc_check.restype = i
    lib.w4a16_gemv_noalloc_timeout_selftest.argtypes = [i, vp]
    lib.w4a16_gemv_noalloc_timeout_selftest.restype = i
    lib.awq_search_workspace_size.argtypes = [i, i, i, i, i]
    lib.awq_search_workspace_size.restype = sz
    lib.awq_search_alpha.argtypes = [vp, vp, i, i, i, vp, i, i, i, i, vp, vp, vp, sz, vp]
    lib.awq_search_alpha.restype = i
    lib.gptq_hessian.argtypes = [vp, i, i, d, vp, vp]
    lib.gptq_hessian.restype = i
    lib.gptq_sweep_workspace_size.argtypes = [i, i, i]
    lib.gptq_sweep_workspace_size.restype = sz
    lib.gptq_sweep.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, vp, sz, vp]
    lib.gptq_sweep.restype = i
    lib.gptq_factor_workspace_size.argtypes = [i]
    lib.gptq_factor_workspace_size.restype = sz
    lib.gptq_factor.argtypes = [vp, i, vp, vp, sz, vp]
    lib.gptq_factor.restype = i
    lib.gptq_quantize_workspace_size.argtypes = [i, i, i]
    lib.gptq_quantize_workspace_size.restype = sz
    lib.gptq_quantize.argtypes = [vp, vp, i, i, i, d, i, i, i, vp, vp, vp, vp, sz, vp]
    lib.gptq_quantize.restype = i
    lib.awq_reference_product.argtypes = [vp, vp, i, i, i, vp, vp]
    lib.awq_reference_product.restype = i
    lib.w4a8_quantize_weight.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp]
    lib.w4a8_quantize_weight.restype = i
    lib.w4a8_quantize_act.argtypes = [vp, i, i, vp, vp, vp]
    lib.w4a8_quantize_act.restype = i
    lib.w4a8_gemm_workspace_size.argtypes = [i, i, i, i]
    lib.w4a8_gemm_workspace_size.restype = sz
    lib.w4a8_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, vp, vp, vp, sz, vp]
    lib.w4a8_gemm.restype = i
    lib.w4a16_gemm_check.argtypes = [vp, vp]
    lib.w4a16_gemm_check.restype = i
    lib.w4a16_wait_timeout_selftest.argtypes = [vp, i, vp]
    lib.w4a16_wait_timeout_selftest.restype = i
    lib.w4a16_last_error.argtypes = []
    lib.w4a16_last_error.restype = ctypes.c_char_p
    lib.w4a16_layout_version.argtypes = []
    lib.w4a16_layout_version.restype = i
    if lib.w4a16_layout_version() != LAYOUT_VERSION:
        raise W4A16Error("libw4a16.so has an unexpected packed-layout version")
    _lib = lib
    return lib


def _check(status: int, name: str) -> None:
    if status != 0:
        msg = load_library().w4a16_last_error().decode(errors="replace")
        raise W4A16Error(f"{name} failed with status {status}: {msg}")


# torch's raw accessors for the current stream and device take a fraction of
# the time of torch.cuda.current_stream / current_device (which build Python
# objects); the public calls are the fallback.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_raw_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(device: torch.device) -> int:
    """The cudaStream_t of the current stream of device, as an integer."""
    if _raw_stream is not None:
        return _raw_stream(device.index)
    return torch.cuda.current_stream(device).cuda_stream


def _current_device() -> int:
    return _raw_device() if _raw_device is not None else torch.cuda.current_device()


def _call_on(device: torch.device, fn, *args) -> int:
    """Runs fn(*args) with device current (the launches go to its streams)."""
    if device.index == _current_device():
        return fn(*args)
    with torch.cuda.device(device):
        return fn(*args)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _expect(t: torch.Tensor, dtype, shape, name: str) -> None:
    # one combined test on the common path; the detailed checks name the fault
    if isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.shape == shape and t.is_contiguous():
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise W4A16Error(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise W4A16Error(f"{name} must have dtype {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise W4A16Error(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise W4A16Error(f"{name} must be contiguous")


def awq_act_scale(X: torch.Tensor, alpha: float = 0.5, out: torch.Tensor | None = None) -> torch.Tensor:
    """s[k] = fp16(mean_t |X[t, k]| ** alpha) for calibration activations X fp16 [T, K]."""
    lib = load_library()
    if X.dim() != 2:
        raise W4A16Error("X must be 2-D [T, K]")
    T, K = X.shape
    _expect(X, torch.float16, (T, K), "X")
    s = torch.empty(K, dtype=torch.float16, device=X.device) if out is None else out
    _expect(s, torch.float16, (K,), "out")
    with torch.cuda.device(X.device):
        _check(lib.awq_act_scale(_ptr(X), T, K, float(alpha), _ptr(s), _stream(X.device)), "awq_act_scale")
    return s


def awq_quantize_pack(W: torch.Tensor, s: torch.Tensor | None = None, group: int = GROUP, bits: int = 4,
                      mode: int = ASYM, out=None):
    """AWQ-scale, group-quantize and pack W fp16 [N, K].

    Returns (qweight int32 [N, K/8] holding uint32 words of layout v1,
    scales fp16 [N, K/group], zeros fp16 [N, K/group]).
    """
    lib = load_library()
    if W.dim() != 2:
        raise W4A16Error("W must be 2-D [N, K]")
    N, K = W.shape
    _expect(W, torch.float16, (N, K), "W")
    if s is not None:
        _expect(s, torch.float16, (K,), "s")
    if group <= 0 or K % group:
        raise W4A16Error(f"K={K} must be a multiple of group={group}")
    if out is None:
        qweight = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
        scales = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
        zeros = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
    else:
        qweight, scales, zeros = out
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(scales, torch.float16, (N, K // group), "scales")
    _expect(zeros, torch.float16, (N, K // group), "zeros")
    with torch.cuda.device(W.device):
        _check(lib.awq_quantize_pack(_ptr(W), _ptr(s), N, K, group, bits, mode, _ptr(qweight), _ptr(scales),
                                     _ptr(zeros), _stream(W.device)), "awq_quantize_pack")
    return qweight, scales, zeros


def gemm_workspace_size(M: int, N: int, K: int, group: int = GROUP) -> int:
    return int(load_library().w4a16_gemm_workspace_size(M, N, K, group))


def workspace_for(device: torch.device, nbytes: int) -> torch.Tensor:
    """A zero-filled workspace of at least nbytes for the current stream of device.

    The kernels leave it zero-filled after every completed call, so one buffer
    per (device, stream) is reused across calls.
    """
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def w4a16_gemm(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
               group: int = GROUP, out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y fp16 [M, N] = x fp16 [M, K] @ dequant(qweight, scales, zeros)^T."""
    lib = _lib if _lib is not None else load_library()
    if x.dim() != 2 or qweight.dim() != 2:
        raise W4A16Error("x must be [M, K] and qweight [N, K/8]")
    M, K = x.shape
    N = qweight.shape[0]
    _expect(x, torch.float16, (M, K), "x")
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(scales, torch.float16, (N, K // group), "scales")
    _expect(zeros, torch.float16, (N, K // group), "zeros")
    y = torch.empty((M, N), dtype=torch.float16, device=x.device) if out is None else out
    _expect(y, torch.float16, (M, N), "out")
    if workspace is None:
        need = gemm_workspace_size(M, N, K, group)
        if need == 0:
            raise W4A16Error(f"unsupported sizes M={M} N={N} K={K} group={group}")
        ws = workspace_for(x.device, need)
    else:
        ws = workspace  # the library checks its size and alignment
    dev = x.device
    _check(_call_on(dev, lib.w4a16_gemm, x.data_ptr(), qweight.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                    M, N, K, group, y.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(), _stream(dev)),
           "w4a16_gemm")
    return y


def w4a16_gemv_noalloc(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                       group: int = GROUP, out: torch.Tensor | None = None) -> torch.Tensor:
    """The split-K GEMV (M <= 4) with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory; ``out`` may be given so
    that this call allocates nothing either.
    """
    lib = load_library()
    M, K = x.shape
    N = qweight.shape[0]
    _expect(x, torch.float16, (M, K), "x")
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(scales, torch.float16, (N, K // group), "scales")
    _expect(zeros, torch.float16, (N, K // group), "zeros")
    y = torch.empty((M, N), dtype=torch.float16, device=x.device) if out is None else out
    _expect(y, torch.float16, (M, N), "out")
    with torch.cuda.device(x.device):
        _check(lib.w4a16_gemv_noalloc(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), M, N, K, group, _ptr(y),
                                      _stream(x.device)), "w4a16_gemv_noalloc")
    return y


def gemv_noalloc_check(device=None) -> None:
    """Synchronizes and raises if a w4a16_gemv_noalloc kernel gave up waiting
    since the last check (the scratch array's status word; cleared here)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib.w4a16_gemv_noalloc_check(_stream(dev)), "w4a16_gemv_noalloc_check")


def gemv_noalloc_timeout_selftest(limit_us: int = 1000, device=None) -> None:
    """Runs the bounded-wait probe on the scratch array's status word (see gemv_noalloc_check)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib.w4a16_gemv_noalloc_timeout_selftest(limit_us, _stream(dev)), "w4a16_gemv_noalloc_timeout_selftest")


def w4a8_quantize_weight(W: torch.Tensor, group: int = GROUP):
    """W fp16 [N, K] -> (qweight int32 [N, K/8] layout v1, s1 fp16 [N], s2 uint8 [N, K/128], zs uint8 [N, K/128])."""
    lib = load_library()
    N, K = W.shape
    _expect(W, torch.float16, (N, K), "W")
    dev = W.device
    q = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
    s1 = torch.empty((N,), dtype=torch.float16, device=dev)
    s2 = torch.empty((N, K // group), dtype=torch.uint8, device=dev)
    zs = torch.empty((N, K // group), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(lib.w4a8_quantize_weight(_ptr(W), N, K, group, _ptr(q), _ptr(s1), _ptr(s2), _ptr(zs), _stream(dev)),
               "w4a8_quantize_weight")
    return q, s1, s2, zs


def w4a8_quantize_act(x: torch.Tensor):
    """x fp16 [M, K] -> (x8 int8 [M, K], s_x fp16 [M])."""
    lib = load_library()
    M, K = x.shape
    _expect(x, torch.float16, (M, K), "x")
    x8 = torch.empty((M, K), dtype=torch.int8, device=x.device)
    sx = torch.empty((M,), dtype=torch.float16, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib.w4a8_quantize_act(_ptr(x), M, K, _ptr(x8), _ptr(sx), _stream(x.device)), "w4a8_quantize_act")
    return x8, sx


def w4a8_gemm_workspace_size(M: int, N: int, K: int, group: int = GROUP) -> int:
    return int(load_library().w4a8_gemm_workspace_size(M, N, K, group))


def w4a8_gemm(x8: torch.Tensor, sx: torch.Tensor, qweight: torch.Tensor, s1: torch.Tensor, s2: torch.Tensor,
              zs: torch.Tensor, group: int = GROUP, out: torch.Tensor | None = None, acc: bool | torch.Tensor = False,
              workspace: torch.Tensor | None = None):
    """y fp16 [M, N] = fp16((acc * s_x) * s1), acc = x8 . (u * s2 - zs)^T exact.

    With acc=True (or an int32 [M, N] tensor) also returns the exact accumulators: (y, acc).
    """
    lib = load_library()
    M, K = x8.shape
    N = qweight.shape[0]
    dev = x8.device
    _expect(x8, torch.int8, (M, K), "x8")
    _expect(sx, torch.float16, (M,), "sx")
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(s1, torch.float16, (N,), "s1")
    _expect(s2, torch.uint8, (N, K // group), "s2")
    _expect(zs, torch.uint8, (N, K // group), "zs")
    y = torch.empty((M, N), dtype=torch.float16, device=dev) if out is None else out
    _expect(y, torch.float16, (M, N), "out")
    acc_t = None
    if isinstance(acc, torch.Tensor):
        acc_t = acc
        _expect(acc_t, torch.int32, (M, N), "acc")
    elif acc:
        acc_t = torch.empty((M, N), dtype=torch.int32, device=dev)
    need = w4a8_gemm_workspace_size(M, N, K, group)
    if workspace is None:
        workspace = workspace_for(dev, need)
    with torch.cuda.device(dev):
        _check(lib.w4a8_gemm(_ptr(x8), _ptr(sx), _ptr(qweight), _ptr(s1), _ptr(s2), _ptr(zs), M, N, K, group,
                             _ptr(y), _ptr(acc_t) if acc_t is not None else None, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(dev)), "w4a8_gemm")
    return (y, acc_t) if acc_t is not None else y


def awq_reference_product(X: torch.Tensor, W: torch.Tensor) -> torch.Tensor:
    """Y fp32 [T, N] = X fp16 [T, K] @ W fp16 [N, K]^T, the alpha search's target (fp32 sums in k order)."""
    lib = load_library()
    T, K = X.shape
    N = W.shape[0]
    _expect(X, torch.float16, (T, K), "X")
    _expect(W, torch.float16, (N, K), "W")
    Y = torch.empty((T, N), dtype=torch.float32, device=X.device)
    with torch.cuda.device(X.device):
        _check(lib.awq_reference_product(_ptr(X), _ptr(W), T, N, K, _ptr(Y), _stream(X.device)), "awq_reference_product")
    return Y


def search_workspace_size(N: int, K: int, T: int, n_alpha: int, group: int = GROUP) -> int:
    return int(load_library().awq_search_workspace_size(N, K, T, n_alpha, group))


def awq_search_alpha(W: torch.Tensor, X: torch.Tensor, alphas, group: int = GROUP, bits: int = 4,
                     mode: int = ASYM, workspace: torch.Tensor | None = None):
    """The AWQ alpha grid search for weights W fp16 [N, K] on calibration tokens X fp16 [T, K].

    Returns (losses, best): the mean squared error of the W4A16 output against
    X W^T for every alpha of the grid, and the index of the smallest.  The call
    waits for the GPU.  ``workspace`` (uint8, any contents) may be given to
    avoid the allocation of search_workspace_size bytes.
    """
    lib = load_library()
    if W.dim() != 2 or X.dim() != 2:
        raise W4A16Error("W must be [N, K] and X [T, K]")
    N, K = W.shape
    T = X.shape[0]
    _expect(W, torch.float16, (N, K), "W")
    _expect(X, torch.float16, (T, K), "X")
    if X.device != W.device:
        raise W4A16Error("W and X must be on the same device")
    grid = [float(a) for a in alphas]
    n = len(grid)
    if workspace is None:
        need = search_workspace_size(N, K, T, n, group)
        if need == 0:
            raise W4A16Error(f"unsupported sizes N={N} K={K} T={T} n_alpha={n} group={group}")
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    elif not isinstance(workspace, torch.Tensor) or workspace.device != W.device:
        raise W4A16Error("workspace must be a tensor on W's device")
    a_buf = (ctypes.c_double * max(n, 1))(*grid)
    losses = (ctypes.c_double * max(n, 1))()
    best = ctypes.c_int(-1)
    with torch.cuda.device(W.device):
        _check(lib.awq_search_alpha(_ptr(W), _ptr(X), N, K, T, a_buf, n, group, bits, mode, losses,
                                    ctypes.byref(best), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(W.device)),
               "awq_search_alpha")
    return [losses[i] for i in range(n)], best.value


def gptq_hessian(X: torch.Tensor, damp: float = 0.01, out: torch.Tensor | None = None) -> torch.Tensor:
    """H fp64 [K, K] = 2 X^T X + damp * mean(diag(2 X^T X)) I for calibration tokens X fp16 [T, K]."""
    lib = load_library()
    if X.dim() != 2:
        raise W4A16Error("X must be 2-D [T, K]")
    T, K = X.shape
    _expect(X, torch.float16, (T, K), "X")
    H = torch.empty((K, K), dtype=torch.float64, device=X.device) if out is None else out
    _expect(H, torch.float64, (K, K), "out")
    with torch.cuda.device(X.device):
        _check(lib.gptq_hessian(_ptr(X), T, K, float(damp), _ptr(H), _stream(X.device)), "gptq_hessian")
    return H


def gptq_sweep(W: torch.Tensor, G: torch.Tensor, group: int = GROUP, bits: int = 4, mode: int = ASYM,
               workspace: torch.Tensor | None = None, out=None):
    """GPTQ's column sweep of W fp16 [N, K] with the upper Cholesky factor G fp64 [K, K] of H^-1.

    Returns (qweight int32 [N, K/8] in layout v1, scales fp16, zeros fp16), as awq_quantize_pack.
    """
    lib = load_library()
    if W.dim() != 2:
        raise W4A16Error("W must be 2-D [N, K]")
    N, K = W.shape
    _expect(W, torch.float16, (N, K), "W")
    _expect(G, torch.float64, (K, K), "G")
    if group <= 0 or K % group:
        raise W4A16Error(f"K={K} must be a multiple of group={group}")
    if out is None:
        qweight = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
        scales = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
        zeros = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
    else:
        qweight, scales, zeros = out
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(scales, torch.float16, (N, K // group), "scales")
    _expect(zeros, torch.float16, (N, K // group), "zeros")
    if workspace is None:
        need = int(lib.gptq_sweep_workspace_size(N, K, group))
        if need == 0:
            raise W4A16Error(f"unsupported sizes N={N} K={K} group={group}")
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib.gptq_sweep(_ptr(W), _ptr(G), N, K, group, bits, mode, _ptr(qweight), _ptr(scales), _ptr(zeros),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(W.device)),
               "gptq_sweep")
    return qweight, scales, zeros


def gptq_factor(H: torch.Tensor, workspace: torch.Tensor | None = None,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """G fp64 [K, K] = Cholesky(H^-1)^T for a symmetric positive definite H fp64 [K, K]."""
    lib = load_library()
    if H.dim() != 2 or H.shape[0] != H.shape[1]:
        raise W4A16Error("H must be square [K, K]")
    K = H.shape[0]
    _expect(H, torch.float64, (K, K), "H")
    G = torch.empty((K, K), dtype=torch.float64, device=H.device) if out is None else out
    _expect(G, torch.float64, (K, K), "out")
    if workspace is None:
        need = int(lib.gptq_factor_workspace_size(K))
        if need == 0:
            raise W4A16Error(f"unsupported size K={K}")
        workspace = torch.empty(need, dtype=torch.uint8, device=H.device)
    with torch.cuda.device(H.device):
        _check(lib.gptq_factor(_ptr(H), K, _ptr(G), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(H.device)), "gptq_factor")
    return G


def gptq_quantize(W: torch.Tensor, X: torch.Tensor, damp: float = 0.01, group: int = GROUP, bits: int = 4,
                  mode: int = ASYM, workspace: torch.Tensor | None = None, out=None):
    """GPTQ of W fp16 [N, K] with calibration tokens X fp16 [T, K]: the Hessian, its factor
    and the column sweep on the GPU.  Returns (qweight int32 [N, K/8] layout v1, scales, zeros)."""
    lib = load_library()
    if W.dim() != 2 or X.dim() != 2:
        raise W4A16Error("W must be [N, K] and X [T, K]")
    N, K = W.shape
    T = X.shape[0]
    _expect(W, torch.float16, (N, K), "W")
    _expect(X, torch.float16, (T, K), "X")
    if group <= 0 or K % group:
        raise W4A16Error(f"K={K} must be a multiple of group={group}")
    if out is None:
        qweight = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
        scales = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
        zeros = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
    else:
        qweight, scales, zeros = out
    _expect(qweight, torch.int32, (N, K // 8), "qweight")
    _expect(scales, torch.float16, (N, K // group), "scales")
    _expect(zeros, torch.float16, (N, K // group), "zeros")
    if workspace is None:
        need = int(lib.gptq_quantize_workspace_size(N, K, group))
        if need == 0:
            raise W4A16Error(f"unsupported sizes N={N} K={K} group={group}")
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib.gptq_quantize(_ptr(W), _ptr(X), N, K, T, float(damp), group, bits, mode, _ptr(qweight),
                                 _ptr(scales), _ptr(zeros), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(W.device)), "gptq_quantize")
    return qweight, scales, zeros


def wait_timeout_selftest(workspace: torch.Tensor, limit_us: int = 1000) -> None:
    """Launches a kernel whose bounded barrier wait runs out after limit_us and
    records the timeout in workspace's status word (see gemm_check)."""
    lib = load_library()
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise W4A16Error("workspace must be a CUDA tensor")
    with torch.cuda.device(workspace.device):
        _check(lib.w4a16_wait_timeout_selftest(_ptr(workspace), limit_us, _stream(workspace.device)),
               "w4a16_wait_timeout_selftest")


def gemm_check(workspace: torch.Tensor) -> None:
    """Synchronizes and raises if a kernel that used this workspace gave up waiting."""
    lib = load_library()
    with torch.cuda.device(workspace.device):
        _check(lib.w4a16_gemm_check(_ptr(workspace), _stream(workspace.device)), "w4a16_gemm_check")
