"""Python binding of the C ABI in include/metis.h (ctypes).

Argument marshalling only: torch tensors provide device memory and the current
CUDA stream; every arithmetic step runs in the CUDA kernels of
``libmetis_b200.so``.  There is no fallback: if the library is missing or the
device is not sm_100, calls raise.
"""
import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmetis_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "metis.h")

OK = 0
BF16, F32 = 0, 1
MXFP4, NVFP4 = 0, 1
SKETCH_GAUSSIAN, SKETCH_SPARSE_SIGN = 0, 1
DEV_NUMERIC, DEV_TIMEOUT, DEV_SAMPLING = 1, 2, 4

FMT = {"mx": MXFP4, "nv": NVFP4, MXFP4: MXFP4, NVFP4: NVFP4}
FMT_NAME = {MXFP4: "mx", NVFP4: "nv"}


class MetisError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        detail = ""
        if status == 6:
            try:
                detail = " [" + lib().metis_last_error().decode() + "]"
            except Exception:  # pragma: no cover
                pass
        super().__init__(f"{what}: {status_string(status)} (status {status}){detail}")


class FP4Struct(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("outer", ctypes.c_int64), ("inner", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("scales_linear", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("inner_sum", ctypes.c_void_p)]


class SplitParams(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("p", ctypes.c_int32), ("power_iters", ctypes.c_int32),
                ("seed", ctypes.c_uint64), ("sketch", ctypes.c_int32),
                ("sparse_nnz", ctypes.c_int32), ("sample_rows", ctypes.c_int64),
                ("fmt", ctypes.c_int32), ("max_core_iters", ctypes.c_int32),
                ("compensate", ctypes.c_int32)]


class OperandStruct(ctypes.Structure):
    _fields_ = [("R", ctypes.POINTER(FP4Struct)), ("k", ctypes.c_int32),
                ("P", ctypes.POINTER(FP4Struct)), ("F", ctypes.POINTER(FP4Struct)),
                ("S", ctypes.c_void_p), ("flags", ctypes.c_int32)]


REQUANT_LOWRANK = 1


_lib = None

_VP, _I32, _I64, _SZP = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)
_FP = ctypes.POINTER(FP4Struct)
_OP = ctypes.POINTER(OperandStruct)

_SIGS = {
    "metis_fp4_codes_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "metis_fp4_scales_bytes": (ctypes.c_size_t, [_I32, _I64, _I64]),
    "metis_status_string": (ctypes.c_char_p, [_I32]),
    "metis_device_supported": (_I32, []),
    "metis_last_error": (ctypes.c_char_p, []),
    "metis_quantize_fp4": (_I32, [_VP, _I32, _I64, _I64, _I64, _I32, _VP, _FP, _VP, _SZP, _VP]),
    "metis_quantize_fp4_noalloc": (_I32, [_VP, _I32, _I64, _I64, _I64, _I32, _VP, _FP, _VP]),
    "metis_noalloc_scratch_bytes": (ctypes.c_size_t, []),
    "metis_selftest_wait_timeout": (_I32, [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "metis_split": (_I32, [_VP, _I32, _I64, _I64, _I64, ctypes.POINTER(SplitParams), _VP, _VP, _VP,
                           _FP, _FP, _FP, _FP, _VP, _VP, _VP, _SZP, _VP, _VP]),
    "metis_linear_fwd": (_I32, [_OP, _OP, _I64, _I64, _I64, _VP, _I32, _I64, _VP, _SZP, _VP, _VP]),
    "metis_linear_bwd": (_I32, [_OP, _OP, _OP, _OP, _I64, _I64, _I64, _VP, _I64, _VP, _I64, _I32,
                                _VP, _SZP, _VP, _VP]),
    "averis_split": (_I32, [_VP, _I32, _I64, _I64, _I64, _I32, _VP, _FP, _FP, _FP, _VP, _VP, _SZP,
                            _VP, _VP]),
    "metis_spectral_scale": (_I32, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _I32, ctypes.c_float, _VP, _VP, _SZP,
                                    _VP, _VP]),
}


def lib():
    """Load libmetis_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmetis_b200.so is not built: run __graft_entry__.build() "
                               "or python spectral_domain_quantization_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions():
    """Names of the functions declared in include/metis.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:METIS_API\s+)?(?:const\s+)?[a-z_0-9]+\s*\**\s+\**(\w+)\s*\(", src,
                                 flags=re.M)))


def status_string(status):
    try:
        return lib().metis_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only when the library is absent
        return "status"


def _check(status, what):
    if status != OK:
        raise MetisError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("only bfloat16 and float32 inputs are supported")


class _Workspace:
    """Grow-only workspace per device and stream (allocated by torch, the
    caller side), so that calls enqueued on different streams never share
    scratch memory."""

    def __init__(self):
        self.buf = {}

    def get(self, nbytes, device):
        key = (torch.device(device).index, torch.cuda.current_stream(device).cuda_stream)
        cur = self.buf.get(key)
        if cur is None or cur.numel() < nbytes:
            cur = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
            self.buf[key] = cur
        return cur


_ws = _Workspace()


def _call_with_workspace(fn, args_before_ws, args_after_ws, device, what, workspace=None):
    """Query the workspace size, provide it (the caller's uint8 tensor when
    given, else the shared per-stream one), then run the call."""
    size = ctypes.c_size_t(0)
    _check(fn(*args_before_ws, None, ctypes.byref(size), *args_after_ws), what + " (workspace query)")
    if workspace is not None:
        if workspace.dtype != torch.uint8 or workspace.numel() < size.value:
            raise ValueError(f"{what}: the workspace needs {size.value} bytes (uint8)")
        ws = workspace
    else:
        ws = _ws.get(size.value, device)
    size2 = ctypes.c_size_t(ws.numel())
    _check(fn(*args_before_ws, _ptr(ws), ctypes.byref(size2), *args_after_ws), what)


# --------------------------------------------------------------------------
# FP4 tensors
# --------------------------------------------------------------------------

class QTensor:
    """An FP4 matrix (outer x inner, blocks along inner) held in torch buffers."""

    def __init__(self, fmt, outer, inner, device="cuda", linear=False, inner_sum=False):
        L = lib()
        self.fmt = FMT[fmt]
        self.outer, self.inner = int(outer), int(inner)
        self.block = 32 if self.fmt == MXFP4 else 16
        self.codes = torch.empty(L.metis_fp4_codes_bytes(self.outer, self.inner), dtype=torch.uint8,
                                 device=device)
        self.scales = torch.empty(L.metis_fp4_scales_bytes(self.fmt, self.outer, self.inner),
                                  dtype=torch.uint8, device=device)
        self.scales_linear = (torch.empty(self.outer * (self.inner // self.block), dtype=torch.uint8,
                                          device=device) if linear else None)
        self.tensor_scale = torch.ones(1, dtype=torch.float32, device=device)
        self.inner_sum = torch.empty(self.outer, dtype=torch.float32, device=device) if inner_sum else None

    def struct(self):
        s = FP4Struct()
        s.fmt, s.outer, s.inner = self.fmt, self.outer, self.inner
        s.codes = self.codes.data_ptr()
        s.scales = self.scales.data_ptr()
        s.scales_linear = self.scales_linear.data_ptr() if self.scales_linear is not None else None
        s.tensor_scale = self.tensor_scale.data_ptr()
        s.inner_sum = self.inner_sum.data_ptr() if self.inner_sum is not None else None
        self._s = s          # keep alive while pointers are in use
        return s


def quantize_fp4(X, fmt, axis=1, sub_col=None, linear=False, inner_sum=False, out=None):
    """FP4 block quantization of a 2-D bf16/f32 CUDA tensor (metis_quantize_fp4)."""
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a row-major 2-D tensor")
    rows, cols = X.shape
    outer, inner = (rows, cols) if axis == 1 else (cols, rows)
    if out is None:
        out = QTensor(fmt, outer, inner, X.device, linear=linear, inner_sum=inner_sum)
    s = out.struct()
    L = lib()
    _call_with_workspace(
        L.metis_quantize_fp4,
        (_ptr(X), _dtype_code(X), rows, cols, X.stride(0), axis, _ptr(sub_col), ctypes.byref(s)),
        (_stream(),), X.device, "metis_quantize_fp4")
    return out


def quantize_fp4_noalloc(X, fmt, axis=1, sub_col=None, linear=False, inner_sum=False, out=None):
    """metis_quantize_fp4_noalloc: the same quantization with the library's
    fixed scratch instead of a workspace (for callers that cannot allocate)."""
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a row-major 2-D tensor")
    rows, cols = X.shape
    outer, inner = (rows, cols) if axis == 1 else (cols, rows)
    if out is None:
        out = QTensor(fmt, outer, inner, X.device, linear=linear, inner_sum=inner_sum)
    s = out.struct()
    _check(lib().metis_quantize_fp4_noalloc(_ptr(X), _dtype_code(X), rows, cols, X.stride(0), axis,
                                            _ptr(sub_col), ctypes.byref(s), _stream()),
           "metis_quantize_fp4_noalloc")
    return out


# --------------------------------------------------------------------------
# split-linear products
# --------------------------------------------------------------------------

class Operand:
    """One operand of an FP4 product (see metis_operand in metis.h).

    left operand  A (M x K) = R + F diag(S) P^T
    right operand B (K x N) = R + P diag(S) F^T
    R: QTensor quantized along K; P: QTensor (outer k, inner K) or None for
    the all-ones vector; F: QTensor (outer k, inner M or N) or None for ones;
    S: CUDA float tensor of k values or None (ones).
    requant: re-quantize the low-rank intermediate formed from this
    operand's factors to FP4 along its k (METIS_REQUANT_LOWRANK)."""

    def __init__(self, R, k=0, P=None, F=None, S=None, requant=False):
        self.R, self.k, self.P, self.F, self.S = R, int(k), P, F, S
        self.requant = bool(requant)

    def struct(self):
        o = OperandStruct()
        self._r = self.R.struct()
        o.R = ctypes.pointer(self._r)
        o.k = self.k
        self._p = self.P.struct() if self.P is not None else None
        self._f = self.F.struct() if self.F is not None else None
        o.P = ctypes.pointer(self._p) if self._p is not None else None
        o.F = ctypes.pointer(self._f) if self._f is not None else None
        o.S = self.S.data_ptr() if self.S is not None else None
        o.flags = REQUANT_LOWRANK if self.requant else 0
        self._o = o
        return o


def _out_dtype(dt):
    return F32 if dt == torch.float32 else BF16


def linear_fwd(X, W, M, N, K, out_dtype=torch.float32, Y=None, dev_status=None):
    """Y = X W on FP4 operands (metis_linear_fwd).  X, W: Operand."""
    dev = X.R.codes.device
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    xs, ws_ = X.struct(), W.struct()
    _call_with_workspace(
        lib().metis_linear_fwd,
        (ctypes.byref(xs), ctypes.byref(ws_), M, N, K, _ptr(Y), _out_dtype(Y.dtype), Y.stride(0)),
        (_ptr(dev_status), _stream()), dev, "metis_linear_fwd")
    return Y


def linear_bwd(dY_n, Wt, Xt, dY_m, M, N, K, out_dtype=torch.float32, dX=None, dW=None,
               want_dx=True, want_dw=True, dev_status=None):
    """dX = dY W^T and dW = X^T dY on FP4 operands (metis_linear_bwd)."""
    dev = (dY_n or Xt).R.codes.device
    if want_dx and dX is None:
        dX = torch.empty((M, K), dtype=out_dtype, device=dev)
    if want_dw and dW is None:
        dW = torch.empty((K, N), dtype=out_dtype, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    a = ctypes.byref(dY_n.struct()) if want_dx else None
    b = ctypes.byref(Wt.struct()) if want_dx else None
    c = ctypes.byref(Xt.struct()) if want_dw else None
    d = ctypes.byref(dY_m.struct()) if want_dw else None
    dt = _out_dtype(out_dtype)
    _call_with_workspace(
        lib().metis_linear_bwd,
        (a, b, c, d, M, N, K, _ptr(dX) if want_dx else None, dX.stride(0) if want_dx else 0,
         _ptr(dW) if want_dw else None, dW.stride(0) if want_dw else 0, dt),
        (_ptr(dev_status), _stream()), dev, "metis_linear_bwd")
    return dX, dW


# --------------------------------------------------------------------------
# spectral split
# --------------------------------------------------------------------------

SKETCH = {"gaussian": SKETCH_GAUSSIAN, "sparse_sign": SKETCH_SPARSE_SIGN}


class Split:
    """Outputs of metis_split: U (m x k), S (k), V (n x k) float32; FP4 U_q
    (k x m), V_q (k x n), R_rows (m x n, blocks along n), R_cols (n x m,
    blocks along m); optional float32 residual tap and sample indices."""

    def __init__(self, **kw):
        self.__dict__.update(kw)

    def operand(self, side, axis_rows=True):
        """Operand of a product: side "right" for W in X W (residual quantized
        along K = rows of W), "left" for X in X W (residual along its columns)."""
        if side == "right":
            return Operand(self.R_cols if axis_rows else self.R_rows, self.k, self.U_q, self.V_q, self.S)
        return Operand(self.R_rows, self.k, self.V_q, self.U_q, self.S)


def split(A, k, p, q=1, seed=0, fmt="nv", sketch="gaussian", nnz=4, sample_rows=0, max_iters=64,
          rows=True, cols=True, factors=True, tap=False, compensate=False, dev_status=None, workspace=None):
    """Spectral split A = U diag(S) V^T + R with FP4 outputs (metis_split).
    compensate: R = A - deq(U_q) diag(S) deq(V_q)^T (needs factors=True).
    workspace: optional caller-owned uint8 CUDA tensor (see sketch_tap)."""
    if A.dim() != 2 or A.stride(1) != 1:
        raise ValueError("A must be a row-major 2-D tensor")
    m, n = A.shape
    dev = A.device
    f = FMT[fmt]
    U = torch.empty((m, k), dtype=torch.float32, device=dev)
    S = torch.empty(k, dtype=torch.float32, device=dev)
    V = torch.empty((n, k), dtype=torch.float32, device=dev)
    U_q = QTensor(f, k, m, dev) if factors else None
    V_q = QTensor(f, k, n, dev) if factors else None
    R_rows = QTensor(f, m, n, dev) if rows else None
    R_cols = QTensor(f, n, m, dev) if cols else None
    R_f32 = torch.empty((m, n), dtype=torch.float32, device=dev) if tap else None
    idx = torch.empty(sample_rows, dtype=torch.int32, device=dev) if sample_rows else None
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    prm = SplitParams(k=k, p=p, power_iters=q, seed=seed, sketch=SKETCH[sketch], sparse_nnz=nnz,
                      sample_rows=sample_rows, fmt=f, max_core_iters=max_iters, compensate=int(bool(compensate)))
    st = [t.struct() if t is not None else None for t in (U_q, V_q, R_rows, R_cols)]
    refs = [ctypes.byref(s) if s is not None else None for s in st]
    _call_with_workspace(
        lib().metis_split,
        (_ptr(A), _dtype_code(A), m, n, A.stride(0), ctypes.byref(prm), _ptr(U), _ptr(S), _ptr(V), *refs,
         _ptr(R_f32), _ptr(idx)),
        (_ptr(dev_status), _stream()), dev, "metis_split", workspace=workspace)
    return Split(U=U, S=S, V=V, U_q=U_q, V_q=V_q, R_rows=R_rows, R_cols=R_cols, R_f32=R_f32, idx=idx,
                 dev_status=dev_status, k=k, fmt=f)


def sketch_tap(workspace, n, k, p):
    """The sketch Omega (n x l, float32 from bf16) that the last metis_split
    on `workspace` used: the first round_up(l, 16) x round_up(n, 8) bf16
    values of the workspace hold Omega^T (the tap metis.h documents)."""
    l = k + p
    lp = (l + 15) // 16 * 16
    ldn = (n + 7) // 8 * 8
    omt = workspace[: lp * ldn * 2].view(torch.bfloat16).view(lp, ldn)
    return omt, omt[:l, :n].float().t()


# --------------------------------------------------------------------------
# Averis
# --------------------------------------------------------------------------

class AverisSplit:
    """Outputs of averis_split: mean (n), mean_q (1 x n), R_rows (m x n,
    blocks along n), R_cols (n x m, blocks along m, with inner sums), tap."""

    def __init__(self, **kw):
        self.__dict__.update(kw)

    def left(self):
        """X as the left operand of X W (contraction over n): 1 mu^T + R."""
        return Operand(self.R_rows, 1, self.mean_q, None, None)

    def left_t(self):
        """X^T as the left operand of X^T dY (contraction over m): mu 1^T + R^T."""
        return Operand(self.R_cols, 1, None, self.mean_q, None)

    def right_m(self):
        """dY as the right operand of X^T dY (contraction over m): 1 nu^T + R."""
        return Operand(self.R_cols, 1, None, self.mean_q, None)


def averis_split(X, fmt="nv", rows=True, cols=True, tap=False, dev_status=None):
    """Mean / residual split with FP4 outputs (averis_split)."""
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a row-major 2-D tensor")
    m, n = X.shape
    dev = X.device
    f = FMT[fmt]
    mean = torch.empty(n, dtype=torch.float32, device=dev)
    mean_q = QTensor(f, 1, n, dev)
    R_rows = QTensor(f, m, n, dev, inner_sum=True) if rows else None
    R_cols = QTensor(f, n, m, dev, inner_sum=True) if cols else None
    R_f32 = torch.empty((m, n), dtype=torch.float32, device=dev) if tap else None
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    st = [t.struct() if t is not None else None for t in (mean_q, R_rows, R_cols)]
    refs = [ctypes.byref(s) if s is not None else None for s in st]
    _call_with_workspace(
        lib().averis_split,
        (_ptr(X), _dtype_code(X), m, n, X.stride(0), f, _ptr(mean), *refs, _ptr(R_f32)),
        (_ptr(dev_status), _stream()), dev, "averis_split")
    return AverisSplit(mean=mean, mean_q=mean_q, R_rows=R_rows, R_cols=R_cols, R_f32=R_f32,
                       dev_status=dev_status, fmt=f)


# --------------------------------------------------------------------------
# mean + spectral composite
# --------------------------------------------------------------------------

class CompositeSplit:
    """A = 1 mu^T + U diag(S) V^T + R2 from averis_split then metis_split of
    the float32 mean-free residual.  The mean and the spectral part form one
    rank-(k + 1) low-rank part F diag(S1) P^T with F = [1 | U], P = [mu | V],
    S1 = [1, S]; F_q (outer k + 1, inner m) and P_q (outer k + 1, inner n) are
    their FP4 quantizations along the long axis.  F32 and P32 are float32
    column views of the factors as quantized (leading dimension padded)."""

    def __init__(self, **kw):
        self.__dict__.update(kw)

    def operand(self, side, axis_rows=True):
        """As Split.operand: "right" for W in X W, "left" for X in X W."""
        if side == "right":
            return Operand(self.R_cols if axis_rows else self.R_rows, self.k1, self.F_q, self.P_q, self.S1)
        return Operand(self.R_rows, self.k1, self.P_q, self.F_q, self.S1)


def composite_split(A, k, p, q=1, seed=0, fmt="nv", sketch="gaussian", nnz=4, max_iters=64,
                    rows=True, cols=True, tap=False, dev_status=None):
    """Mean removal (averis_split, float32 residual tap) followed by the
    spectral split of the residual (metis_split), then the FP4 factors of the
    rank-(k + 1) low-rank part (metis_quantize_fp4).  Every step runs in the
    library's kernels; this function only arranges buffers."""
    if A.dim() != 2 or A.stride(1) != 1:
        raise ValueError("A must be a row-major 2-D tensor")
    m, n = A.shape
    dev = A.device
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    av = averis_split(A, fmt, rows=False, cols=False, tap=True, dev_status=dev_status)
    sp = split(av.R_f32, k, p, q, seed, fmt, sketch=sketch, nnz=nnz, max_iters=max_iters, rows=rows,
               cols=cols, factors=False, tap=tap, dev_status=dev_status)
    k1 = k + 1
    ldk = (k1 + 3) // 4 * 4                     # rows start on 16-byte boundaries
    Fbuf = torch.zeros((m, ldk), dtype=torch.float32, device=dev)
    Pbuf = torch.zeros((n, ldk), dtype=torch.float32, device=dev)
    Fbuf[:, 0] = 1.0
    Fbuf[:, 1:k1] = sp.U
    Pbuf[:, 0] = av.mean
    Pbuf[:, 1:k1] = sp.V
    F32, P32 = Fbuf[:, :k1], Pbuf[:, :k1]
    F_q = quantize_fp4(F32, fmt, 0)
    P_q = quantize_fp4(P32, fmt, 0)
    S1 = torch.cat([torch.ones(1, dtype=torch.float32, device=dev), sp.S])
    return CompositeSplit(mean=av.mean, R1=av.R_f32, U=sp.U, S=sp.S, V=sp.V, F32=F32, P32=P32, F_q=F_q,
                          P_q=P_q, S1=S1, R_rows=sp.R_rows, R_cols=sp.R_cols, R2_f32=sp.R_f32, k=k, k1=k1,
                          fmt=sp.fmt, dev_status=dev_status)


def spectral_scale(G, U, S, V, cap, out=None, dev_status=None):
    """Adaptive spectral learning (metis_spectral_scale): G' = P_L G P_R with
    the gains min(S_1 / S_i, cap) along the split's singular directions.
    G: K x N float32 CUDA tensor; U (K x k), S (k), V (N x k) from split()."""
    if G.dim() != 2 or G.stride(1) != 1 or G.dtype != torch.float32:
        raise ValueError("G must be a row-major float32 2-D tensor")
    if not (U.is_contiguous() and S.is_contiguous() and V.is_contiguous()):
        raise ValueError("U, S and V must be contiguous")
    K, N = G.shape
    k = U.shape[1]
    if out is None:
        out = torch.empty((K, N), dtype=torch.float32, device=G.device)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=G.device)
    _call_with_workspace(
        lib().metis_spectral_scale,
        (_ptr(G), K, N, G.stride(0), _ptr(U), _ptr(S), _ptr(V), k,
         ctypes.c_float(cap), _ptr(out)),
        (_ptr(dev_status), _stream()), G.device, "metis_spectral_scale")
    return out


def selftest_wait_timeout(limit_ns=1_000_000, device="cuda"):
    """Run the library's bounded device wait on a barrier that never
    completes (metis_selftest_wait_timeout); returns the device status word
    after the launch finished (DEV_TIMEOUT set when the wait ended itself)."""
    st = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib().metis_selftest_wait_timeout(int(limit_ns), _ptr(st), _stream()), "metis_selftest_wait_timeout")
    torch.cuda.synchronize()
    return int(st.item())
