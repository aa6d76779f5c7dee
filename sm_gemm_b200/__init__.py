"""Python binding of the smgemm C-ABI (libsmgemm.so, built for sm_100a).

Argument marshalling only: torch tensors give device pointers, leading dimensions
and the current CUDA stream; every computation runs in the library's kernels. Before a
call, every tensor is checked to be on the call's CUDA device with the type and shape
the sizes imply (ValueError otherwise), since the kernels dereference what they are
given. There is no fallback: if the library is missing or a call fails, an exception
is raised.

    import sm_gemm_b200 as sg
    C = sg.gemm_bf16(A, B, bias=b, act="gelu_tanh", out_dtype=torch.bfloat16)
    Q, S = sg.quantize_fp8_blockwise(X, group_rows=1)
    C = sg.gemm_fp8_blockscaled(Aq, sa, Bq, sb, out_dtype=torch.bfloat16)
    Cs = sg.gemm_bf16_grouped([A0, A1], [B0, B1])
"""
from __future__ import annotations

import ctypes as C
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmgemm.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
F32, BF16, F16, E4M3 = 0, 1, 2, 3
ROW_MAJOR, COL_MAJOR = 0, 1
ACTS = {"none": 0, None: 0, "gelu_tanh": 1, "gelu": 1, "silu": 2}

_lock = threading.Lock()
_lib = None
_ws_cache: dict = {}
_ws_retired: list = []


class SmgemmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"smgemm {what}: status {status} ({status_string(status)})")


def lib():
    """The loaded C library (built in-tree by ``python -m sm_gemm_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sm_gemm_b200.build`")
            L = C.CDLL(LIB_PATH)
            I64, P, I, SZ = C.c_int64, C.c_void_p, C.c_int, C.c_size_t
            L.gemm_bf16.argtypes = [I64, I64, I64, P, I, I, I64, P, I, I64, P, I, I, P, I, I64, P, SZ, P]
            L.gemm_bf16.restype = I
            L.gemm_fp8_blockscaled.argtypes = [I64, I64, I64, P, P, P, P, P, I, I, P, I, I64, P, SZ, P]
            L.gemm_fp8_blockscaled.restype = I
            L.quantize_fp8_blockwise.argtypes = [P, I64, I64, I, I64, I, P, P, P]
            L.quantize_fp8_blockwise.restype = I
            L.smgemm_workspace_size.argtypes = [I64, I64, I64, I]
            L.smgemm_workspace_size.restype = SZ
            L.smgemm_status_string.argtypes = [I]
            L.smgemm_status_string.restype = C.c_char_p
            L.smgemm_check.argtypes = [P]
            L.smgemm_check.restype = I
            L.smgemm_last_config.argtypes = []
            L.smgemm_last_config.restype = C.c_char_p
            L.smgemm_selftest_wait_timeout.argtypes = [C.c_uint32, P]
            L.smgemm_selftest_wait_timeout.restype = I
            L.smgemm_schedule_dump.argtypes = [I64, I64, I64, I, I, I, P, I64]
            L.smgemm_schedule_dump.restype = I64
            PI64, PP = C.POINTER(C.c_int64), C.POINTER(C.c_void_p)
            L.gemm_bf16_grouped.argtypes = [I, PI64, PI64, PI64, PP, I, I, PI64, PP, I, PI64, PP, I, I, PP, I,
                                            PI64, P, SZ, P]
            L.gemm_bf16_grouped.restype = I
            L.smgemm_grouped_workspace_size.argtypes = [I]
            L.smgemm_grouped_workspace_size.restype = SZ
            L.gemm_bf16_logsoftmax.argtypes = [I64, I64, I64, P, I, I, I64, P, I, I64, P, I, P, I64, P, SZ, P]
            L.gemm_bf16_logsoftmax.restype = I
            L.smgemm_logsoftmax_workspace_size.argtypes = [I64, I64, I64]
            L.smgemm_logsoftmax_workspace_size.restype = SZ
            L.gemm_bf16_fp8out.argtypes = [I64, I64, I64, P, I, I, I64, P, I, I64, P, I, I, P, I64, P, P, SZ, P]
            L.gemm_bf16_fp8out.restype = I
            L.gemm_bf16_lse_partials.argtypes = [I64, I64, I64, P, I, I, I64, P, I, I64, P, I, P, I64, P, P, SZ, P]
            L.gemm_bf16_lse_partials.restype = I
            L.logsoftmax_apply_partials.argtypes = [P, I64, I64, I64, P, I64, P, P]
            L.logsoftmax_apply_partials.restype = I
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().smgemm_status_string(status).decode()


def _torch():
    import torch
    return torch


_DTYPES: dict = {}


def _dtype_code(dt) -> int:
    if not _DTYPES:
        torch = _torch()
        _DTYPES.update({torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16})
    code = _DTYPES.get(dt)
    if code is None:
        raise ValueError(f"unsupported dtype {dt} (float32, bfloat16 or float16)")
    return code


# Host-side checks of every tensor a call hands to the library: the kernels dereference
# the pointers they are given, so a host tensor, a tensor on another GPU, or one smaller
# than the sizes say must be refused here rather than read or written out of bounds.

def _need(ok: bool, msg: str):
    if not ok:
        raise ValueError(msg)


def _device(*ts):
    """CUDA device index shared by the given tensors (None entries are skipped)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        _need(t.is_cuda, "every tensor of a call must be on a CUDA device")
        d = t.get_device()
        _need(dev is None or d == dev, "all tensors of a call must be on one CUDA device")
        dev = d
    return dev


_getdev = None


def _current_device():
    """Index of the current CUDA device (torch's raw getter once torch is initialised)."""
    global _getdev
    if _getdev is None:
        torch = _torch()
        torch.cuda.init()
        _getdev = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device
    return _getdev()


# The checks below build their error messages only when a check fails: they run on
# every call, and formatting a message costs as much as the check itself.

def _shape(t, want, name):
    if tuple(t.shape) != tuple(want):
        raise ValueError(f"{name} must have shape {tuple(want)}, not {tuple(t.shape)}")


def _dense(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _vector(t, n, name):
    """A bias: 1-D, unit stride, at least n elements."""
    if not (t.dim() == 1 and t.shape[0] >= n and (t.shape[0] <= 1 or t.stride(0) == 1)):
        raise ValueError(f"{name} must be a unit-stride vector of at least {n} elements")
    _dtype_code(t.dtype)


def _out_matrix(t, M, N, name, dtypes=None):
    _shape(t, (M, N), name)
    if not (t.dim() == 2 and (t.stride(1) == 1 or N <= 1)):
        raise ValueError(f"{name} must be row-major")
    if dtypes is not None:
        if t.dtype not in dtypes:
            raise ValueError(f"{name} must be one of {dtypes}")
    else:
        _dtype_code(t.dtype)


def _ldc(out, M, N):
    """Row pitch of an output. A single row's pitch is never used to address anything,
    so it is rounded up to 16 elements (16-byte aligned for every output type) instead
    of failing the library's pitch-alignment check (a one-token LM head with an odd
    vocabulary size)."""
    ld = max(out.stride(0), N)
    return -(-ld // 16) * 16 if M == 1 else ld


def _ws_bytes(workspace):
    _dense(workspace, "workspace")
    return workspace.numel() * workspace.element_size()


def _layout(t, name):
    """(layout, leading dimension) of a 2-D tensor; one of its strides must be 1."""
    st = t.stride()
    if len(st) != 2:
        raise ValueError(f"{name} must be 2-D")
    (rows, cols), (s0, s1) = t.shape, st
    if rows == 0 or cols == 0:
        # nothing is read; any strides (numpy gives an empty array zero strides)
        return ROW_MAJOR, -(-max(cols, 1) // 8) * 8
    if s1 == 1 and (rows <= 1 or s0 >= cols):
        return ROW_MAJOR, max(s0, cols)
    if s0 == 1:
        return COL_MAJOR, max(s1, rows)
    raise ValueError(f"{name} must have a unit stride in one dimension")


def _layout_as(t, name, want, g=None):
    """Leading dimension of a 2-D tensor read in layout `want` (grouped calls share one
    layout): a single row or column fits either layout, and its unused leading
    dimension is rounded up to 8 elements (16 bytes). `g` (a group index) is only used
    in the error message."""
    rows, cols = t.shape
    s0, s1 = t.stride()
    if rows == 0 or cols == 0:  # nothing is read: any strides, a 16-byte leading dimension
        return -(-max(cols if want == ROW_MAJOR else rows, 1) // 8) * 8
    if want == ROW_MAJOR and (s1 == 1 or cols <= 1):
        return max(s0, cols) if rows > 1 else -(-max(cols, 1) // 8) * 8
    if want == COL_MAJOR and (s0 == 1 or rows <= 1):
        return max(s1, rows) if cols > 1 else -(-max(rows, 1) // 8) * 8
    raise ValueError(f"{name}{'' if g is None else f'[{g}]'} cannot be read in the layout the other groups use")


_current_stream = None


def _stream(stream):
    """The cudaStream_t handle of `stream` (a torch stream or a raw handle), or of
    torch's current stream on the current device when None."""
    global _current_stream
    if stream is None:
        if _current_stream is None:
            torch = _torch()
            torch.cuda.init()
            getdev = getattr(torch._C, "_cuda_getDevice", None)
            raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
            if getdev is not None and raw is not None:
                _current_stream = lambda: raw(getdev())
            else:
                _current_stream = lambda: torch.cuda.current_stream().cuda_stream
        return _current_stream()
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return stream


def _workspace(nbytes: int, device, stream_handle):
    """A cached workspace of at least nbytes for calls on (device, stream). Calls on one
    stream run in order and share it; calls on different streams, which may overlap,
    get different ones. A workspace that is outgrown is kept alive (in _ws_retired),
    since kernels already queued may still use it; sizes at least double, so the kept
    ones total less than the live one."""
    if nbytes == 0:
        return None, 0
    torch = _torch()
    key = (device.index if device.index is not None else torch.cuda.current_device(),
           int(getattr(stream_handle, "value", stream_handle) or 0))
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        if ws is not None:
            _ws_retired.append(ws)
        size = max(nbytes, 1 << 20, 0 if ws is None else 2 * ws.numel())
        ws = torch.empty(size, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws, ws.numel()


def _check(status: int, what: str):
    if status != OK:
        raise SmgemmError(status, what)


def workspace_size(M: int, N: int, K: int, kind: int = 0) -> int:
    return int(lib().smgemm_workspace_size(M, N, K, kind))


def gemm_bf16(A, B, *, bias=None, act="none", out=None, out_dtype=None, workspace=None, stream=None):
    """C = act(A @ B + bias) for bf16/f16 A[M,K], B[K,N] (any unit-stride layout).

    ``out`` (row-major [M,N]) is allocated when not given; ``out_dtype`` defaults to
    A's dtype. Returns ``out``."""
    dev = _device(A, B, bias, out, workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_bf16(A, B, bias=bias, act=act, out=out, out_dtype=out_dtype, workspace=workspace,
                             stream=stream)
    torch = _torch()
    M, K = A.shape
    K2, N = B.shape
    if K != K2 or A.dtype != B.dtype:
        raise ValueError("A and B must agree in K and dtype")
    la, lda = _layout(A, "A")
    lb, ldb = _layout(B, "B")
    if bias is not None:
        _vector(bias, N, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A.dtype, device=A.device)
    _out_matrix(out, M, N, "out")
    ldc = _ldc(out, M, N)
    sh = _stream(stream)
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else \
        _workspace(workspace_size(M, N, K, 0), A.device, sh)
    st = lib().gemm_bf16(M, N, K, A.data_ptr(), _dtype_code(A.dtype), la, lda, B.data_ptr(), lb, ldb,
                         None if bias is None else bias.data_ptr(),
                         _dtype_code(bias.dtype) if bias is not None else 0, ACTS[act],
                         out.data_ptr(), _dtype_code(out.dtype), ldc,
                         None if ws is None else ws.data_ptr(), wsb, sh)
    _check(st, "gemm_bf16")
    return out


def gemm_bf16_fp8out(A, B, *, bias=None, act="none", Q=None, scales=None, workspace=None, stream=None):
    """act(A @ B + bias) quantised to E4M3 with one FP32 scale per 1x128 row group:
    returns (codes uint8 [M, N], scales float32 [ceil(N/128), M]), the A operand of
    gemm_fp8_blockscaled."""
    dev = _device(A, B, bias, Q, scales, workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_bf16_fp8out(A, B, bias=bias, act=act, Q=Q, scales=scales, workspace=workspace,
                                    stream=stream)
    torch = _torch()
    M, K = A.shape
    K2, N = B.shape
    if K != K2 or A.dtype != B.dtype:
        raise ValueError("A and B must agree in K and dtype")
    la, lda = _layout(A, "A")
    lb, ldb = _layout(B, "B")
    if bias is not None:
        _vector(bias, N, "bias")
    if Q is None:
        Q = torch.empty((M, -(-N // 16) * 16), dtype=torch.uint8, device=A.device)[:, :N]
    if scales is None:
        scales = torch.empty((-(-N // 128), M), dtype=torch.float32, device=A.device)
    _out_matrix(Q, M, N, "Q", (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)))
    _shape(scales, (-(-N // 128), M), "scales")
    _dense(scales, "scales")
    _need(scales.dtype == torch.float32, "scales must be float32")
    ldc = _ldc(Q, M, N)
    sh = _stream(stream)
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else \
        _workspace(workspace_size(M, N, K, 0), A.device, sh)
    st = lib().gemm_bf16_fp8out(M, N, K, A.data_ptr(), _dtype_code(A.dtype), la, lda, B.data_ptr(), lb, ldb,
                                None if bias is None else bias.data_ptr(),
                                _dtype_code(bias.dtype) if bias is not None else 0, ACTS[act],
                                Q.data_ptr(), ldc, scales.data_ptr(), None if ws is None else ws.data_ptr(), wsb,
                                sh)
    _check(st, "gemm_bf16_fp8out")
    return Q, scales


def gemm_bf16_logsoftmax(A, B, *, bias=None, out=None, workspace=None, stream=None):
    """log_softmax(A @ B + bias) over each row, FP32 [M, N] (the LM head and its
    log-softmax, fused). A, B, bias as in gemm_bf16; ``out`` is allocated if not given."""
    dev = _device(A, B, bias, out, workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_bf16_logsoftmax(A, B, bias=bias, out=out, workspace=workspace, stream=stream)
    torch = _torch()
    M, K = A.shape
    K2, N = B.shape
    if K != K2 or A.dtype != B.dtype:
        raise ValueError("A and B must agree in K and dtype")
    la, lda = _layout(A, "A")
    lb, ldb = _layout(B, "B")
    if bias is not None:
        _vector(bias, N, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _out_matrix(out, M, N, "out", (torch.float32,))
    ldc = _ldc(out, M, N)
    sh = _stream(stream)
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else \
        _workspace(int(lib().smgemm_logsoftmax_workspace_size(M, N, K)), A.device, sh)
    st = lib().gemm_bf16_logsoftmax(M, N, K, A.data_ptr(), _dtype_code(A.dtype), la, lda, B.data_ptr(), lb, ldb,
                                    None if bias is None else bias.data_ptr(),
                                    _dtype_code(bias.dtype) if bias is not None else 0,
                                    out.data_ptr(), ldc, None if ws is None else ws.data_ptr(), wsb, sh)
    _check(st, "gemm_bf16_logsoftmax")
    return out


def gemm_bf16_lse_partials(A, B, *, bias=None, out=None, part=None, workspace=None, stream=None):
    """Logits z = A @ B + bias (FP32 [M, N]) and, per 128-column tile t and row m, the pair
    (max z, sum exp(z - max)) in part[t, m] (float32 [ceil(N/128), M, 2]): the first step of
    a vocabulary-parallel log-softmax. Returns (out, part)."""
    dev = _device(A, B, bias, out, part, workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_bf16_lse_partials(A, B, bias=bias, out=out, part=part, workspace=workspace, stream=stream)
    torch = _torch()
    M, K = A.shape
    K2, N = B.shape
    if K != K2 or A.dtype != B.dtype:
        raise ValueError("A and B must agree in K and dtype")
    la, lda = _layout(A, "A")
    lb, ldb = _layout(B, "B")
    if bias is not None:
        _vector(bias, N, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _out_matrix(out, M, N, "out", (torch.float32,))
    if part is None:
        part = torch.empty((-(-N // 128), M, 2), dtype=torch.float32, device=A.device)
    _shape(part, (-(-N // 128), M, 2), "part")
    _dense(part, "part")
    _need(part.dtype == torch.float32, "part must be float32")
    ldc = _ldc(out, M, N)
    sh = _stream(stream)
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else \
        _workspace(workspace_size(M, N, K, 0), A.device, sh)
    st = lib().gemm_bf16_lse_partials(M, N, K, A.data_ptr(), _dtype_code(A.dtype), la, lda, B.data_ptr(), lb, ldb,
                                      None if bias is None else bias.data_ptr(),
                                      _dtype_code(bias.dtype) if bias is not None else 0,
                                      out.data_ptr(), ldc, part.data_ptr(), None if ws is None else ws.data_ptr(),
                                      wsb, sh)
    _check(st, "gemm_bf16_lse_partials")
    return out, part


def logsoftmax_apply_partials(C, part, *, lse=None, stream=None):
    """lse[m] merged from every pair part[p, m] (float32 [P, M, 2], e.g. all ranks' partials
    stacked), then C[m, n] -= lse[m] in place (C: FP32 [M, N], N may be 0). Returns lse."""
    dev = _device(C, part, lse)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return logsoftmax_apply_partials(C, part, lse=lse, stream=stream)
    torch = _torch()
    M, N = C.shape
    _need(part.dim() == 3 and part.shape[1] == M and part.shape[2] == 2, "part must be [P, M, 2]")
    _dense(part, "part")
    _need(part.dtype == torch.float32 and part.shape[0] >= 1, "part must be float32 with P >= 1")
    if lse is None:
        lse = torch.empty((M,), dtype=torch.float32, device=C.device)
    _vector(lse, M, "lse")
    _need(lse.dtype == torch.float32 and lse.is_contiguous(), "lse must be a contiguous float32 vector")
    _out_matrix(C, M, N, "C", (torch.float32,))
    ldc = _ldc(C, M, N)
    st = lib().logsoftmax_apply_partials(C.data_ptr(), ldc, M, N, part.data_ptr(), part.shape[0], lse.data_ptr(),
                                         _stream(stream))
    _check(st, "logsoftmax_apply_partials")
    return lse


def gemm_bf16_grouped(As, Bs, *, biases=None, act="none", outs=None, out_dtype=None, workspace=None,
                      stream=None):
    """C_g = act(A_g @ B_g + bias_g) for every group g in one launch. All A_g share one
    layout and dtype, all B_g one layout; sizes may differ. ``outs`` (row-major) are
    allocated when not given. Returns the list of outputs."""
    G = len(As)
    if len(Bs) != G or (biases is not None and len(biases) != G) or (outs is not None and len(outs) != G):
        raise ValueError("As, Bs, biases and outs must have one entry per group")
    if G == 0:
        return []
    dev = _device(*As, *Bs, *(biases or ()), *(outs or ()), workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_bf16_grouped(As, Bs, biases=biases, act=act, outs=outs, out_dtype=out_dtype,
                                     workspace=workspace, stream=stream)
    args, res = _grouped_marshal(As, Bs, biases, act, outs, out_dtype, workspace, _stream(stream))
    _check(lib().gemm_bf16_grouped(*args), "gemm_bf16_grouped")
    return res


def _grouped_marshal(As, Bs, biases, act, outs, out_dtype, workspace, sh):
    """Checks every group and builds gemm_bf16_grouped's arguments (stream handle `sh`
    last); allocates missing outputs and the workspace. Returns (args, outputs). It reads
    each tensor's shape, strides and pointer once: with many small groups (MoE experts at
    decode sizes) this marshalling is most of a call's host time."""
    G = len(As)
    torch = _torch()
    adt = As[0].dtype
    # The shared layouts: those of the first group whose operand is not a single row or column.
    lay_a = next((_layout(A, "A")[0] for A in As if min(A.shape) > 1), ROW_MAJOR)
    lay_b = next((_layout(B, "B")[0] for B in Bs if min(B.shape) > 1), ROW_MAJOR)
    Ms, Ns, Ks, ldas, ldbs, ldcs = [0] * G, [0] * G, [0] * G, [0] * G, [0] * G, [0] * G
    pA, pB, pC = [0] * G, [0] * G, [0] * G
    res = outs if outs is not None else [None] * G
    cdt = None
    for g in range(G):
        A, B = As[g], Bs[g]
        M, K = A.shape
        K2, N = B.shape
        if K != K2 or A.dtype is not adt or B.dtype is not adt:
            raise ValueError(f"group {g}: A and B must agree in K and dtype")
        ldas[g] = _layout_as(A, "A", lay_a, g)
        ldbs[g] = _layout_as(B, "B", lay_b, g)
        if biases is not None and biases[g] is not None:
            _vector(biases[g], N, f"biases[{g}]")
        out = res[g]
        if out is None:
            out = torch.empty((M, N), dtype=out_dtype or adt, device=A.device)
            res[g] = out
        oshape, ostride = out.shape, out.stride()
        if len(oshape) != 2 or oshape[0] != M or oshape[1] != N or not (ostride[1] == 1 or N <= 1):
            _out_matrix(out, M, N, f"outs[{g}]")          # raises the precise error
        if cdt is None:
            cdt = out.dtype
            _dtype_code(cdt)
        elif out.dtype is not cdt:
            raise ValueError("outputs must share one dtype")
        ld = max(ostride[0], N)
        ldcs[g] = -(-ld // 16) * 16 if M == 1 else ld
        Ms[g], Ns[g], Ks[g] = M, N, K
        pA[g], pB[g], pC[g] = A.data_ptr(), B.data_ptr(), out.data_ptr()
    I64G, PG = C.c_int64 * G, C.c_void_p * G
    nbytes = int(lib().smgemm_grouped_workspace_size(G))
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else _workspace(nbytes, As[0].device, sh)
    bias_dt, pbias = 0, None
    if biases is not None:
        bias_dt = next((_dtype_code(b.dtype) for b in biases if b is not None), 0)
        _need(all(b is None or _dtype_code(b.dtype) == bias_dt for b in biases), "biases must share one dtype")
        pbias = PG(*[None if b is None else b.data_ptr() for b in biases])
    args = (G, I64G(*Ms), I64G(*Ns), I64G(*Ks), PG(*pA), _dtype_code(adt), lay_a, I64G(*ldas), PG(*pB), lay_b,
            I64G(*ldbs), pbias, bias_dt, ACTS[act], PG(*pC), _dtype_code(cdt), I64G(*ldcs),
            None if ws is None else ws.data_ptr(), wsb, sh)
    return args, list(res)


class GroupedGemm:
    """A grouped GEMM prepared once and launched many times: the tensors are checked and
    the argument arrays of gemm_bf16_grouped built in the constructor, so each call only
    enqueues the launch (the host time of a call with many small groups - MoE experts at
    decode sizes - is then the library's own, not the argument marshalling). The tensors
    must keep their storage, shapes and strides (their contents may change) for as long
    as the object is used; the object holds references to them.

        g = GroupedGemm(As, Bs, biases=None, act="none", outs=None, out_dtype=None, workspace=None)
        g()                # or g(stream=s); returns the outputs
    """

    def __init__(self, As, Bs, *, biases=None, act="none", outs=None, out_dtype=None, workspace=None):
        torch = _torch()
        G = len(As)
        if len(Bs) != G or (biases is not None and len(biases) != G) or (outs is not None and len(outs) != G):
            raise ValueError("As, Bs, biases and outs must have one entry per group")
        if G == 0:
            raise ValueError("a grouped GEMM needs at least one group")
        self.device = _device(*As, *Bs, *(biases or ()), *(outs or ()), workspace)
        if workspace is None:   # its own workspace: calls on different streams may overlap
            workspace = torch.empty(max(int(lib().smgemm_grouped_workspace_size(G)), 16), dtype=torch.uint8,
                                    device=As[0].device)
        args, self.outs = _grouped_marshal(As, Bs, biases, act, outs, out_dtype, workspace, 0)
        self._args = list(args)
        self._keep = (list(As), list(Bs), list(biases or ()), workspace)

    def __call__(self, stream=None):
        if self.device != _current_device():
            with _torch().cuda.device(self.device):
                return self(stream)
        self._args[-1] = _stream(stream)
        _check(lib().gemm_bf16_grouped(*self._args), "gemm_bf16_grouped")
        return self.outs


def gemm_fp8_blockscaled(Aq, sa, Bq, sb, *, bias=None, act="none", out=None, out_dtype=None,
                         workspace=None, stream=None):
    """C = act(sum_kb sa*sb*(Aq @ Bq^T)_kb + bias) from E4M3 codes Aq[M,K], Bq[N,K] (uint8 or
    float8_e4m3fn, K contiguous) and FP32 scales sa[KB,M], sb[KB,NB]."""
    dev = _device(Aq, sa, Bq, sb, bias, out, workspace)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return gemm_fp8_blockscaled(Aq, sa, Bq, sb, bias=bias, act=act, out=out, out_dtype=out_dtype,
                                        workspace=workspace, stream=stream)
    torch = _torch()
    M, K = Aq.shape
    N, K2 = Bq.shape
    if K != K2:
        raise ValueError("Aq and Bq must agree in K")
    for t, n in ((Aq, "Aq"), (Bq, "Bq"), (sa, "sa"), (sb, "sb")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    codes = (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8))
    _need(Aq.dtype in codes and Bq.dtype in codes, "Aq and Bq must be uint8 or float8_e4m3fn codes")
    _need(sa.dtype == torch.float32 and sb.dtype == torch.float32, "sa and sb must be float32")
    _shape(sa, (-(-K // 128), M), "sa")
    _shape(sb, (-(-K // 128), -(-N // 128)), "sb")
    if bias is not None:
        _vector(bias, N, "bias")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=Aq.device)
    _out_matrix(out, M, N, "out")
    ldc = _ldc(out, M, N)
    sh = _stream(stream)
    ws, wsb = (workspace, _ws_bytes(workspace)) if workspace is not None else \
        _workspace(workspace_size(M, N, K, 1), Aq.device, sh)
    st = lib().gemm_fp8_blockscaled(M, N, K, Aq.data_ptr(), sa.data_ptr(), Bq.data_ptr(), sb.data_ptr(),
                                    None if bias is None else bias.data_ptr(),
                                    _dtype_code(bias.dtype) if bias is not None else 0, ACTS[act],
                                    out.data_ptr(), _dtype_code(out.dtype), ldc,
                                    None if ws is None else ws.data_ptr(), wsb, sh)
    _check(st, "gemm_fp8_blockscaled")
    return out


def quantize_fp8_blockwise(X, group_rows: int = 1, *, Q=None, scales=None, stream=None):
    """FP32 X[rows, cols] -> (codes uint8, scales float32). group_rows=1: 1x128 groups,
    codes [rows, cols], scales [ceil(cols/128), rows]. group_rows=128: 128x128 blocks of
    the weight X[K, N], codes written transposed [N, K], scales [ceil(K/128), ceil(N/128)]."""
    dev = _device(X, Q, scales)
    if dev != _current_device():
        with _torch().cuda.device(dev):
            return quantize_fp8_blockwise(X, group_rows, Q=Q, scales=scales, stream=stream)
    torch = _torch()
    _need(X.dtype == torch.float32, "X must be float32")
    rows, cols = X.shape
    lx, ldx = _layout(X, "X")
    if group_rows == 1:
        qshape, sshape = (rows, cols), (-(-cols // 128), rows)
    else:
        qshape, sshape = (cols, rows), (-(-rows // 128), -(-cols // 128))
    if Q is None:
        Q = torch.empty(qshape, dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(sshape, dtype=torch.float32, device=X.device)
    _shape(Q, qshape, "Q")
    _dense(Q, "Q")
    _need(Q.dtype in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)), "Q must hold uint8 codes")
    _shape(scales, sshape, "scales")
    _dense(scales, "scales")
    _need(scales.dtype == torch.float32, "scales must be float32")
    st = lib().quantize_fp8_blockwise(X.data_ptr(), rows, cols, lx, ldx, group_rows, Q.data_ptr(),
                                      scales.data_ptr(), _stream(stream))
    _check(st, "quantize_fp8_blockwise")
    return Q, scales


def check(stream=None) -> int:
    """Synchronise the stream and return the library status (ERR_TIMEOUT if a kernel
    abandoned a barrier wait since the last check)."""
    return int(lib().smgemm_check(_stream(stream)))


def last_config() -> str:
    return lib().smgemm_last_config().decode()


def selftest_wait_timeout(limit_us: int, stream=None) -> int:
    return int(lib().smgemm_selftest_wait_timeout(limit_us, _stream(stream)))


def schedule_dump(M: int, N: int, K: int, kind: int = 0, layout_a: int = ROW_MAJOR, num_sms: int = 148):
    """Segments (cta, tile, m_tile, n_tile, kb_begin, kb_end, slot) of the persistent
    schedule a call with these sizes uses on a GPU with ``num_sms`` SMs (host only)."""
    import numpy as np
    n = lib().smgemm_schedule_dump(M, N, K, kind, layout_a, num_sms, None, 0)
    out = np.zeros((max(n, 1), 7), dtype=np.int32)
    lib().smgemm_schedule_dump(M, N, K, kind, layout_a, num_sms, out.ctypes.data_as(C.c_void_p), n)
    return out[:n]
