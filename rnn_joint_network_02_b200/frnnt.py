"""Thin Python binding of libfrnnt.so (ctypes).

Argument marshalling only: every step of the forward and backward pass runs
in the library's CUDA kernels.  PyTorch supplies device memory and the
stream.  If the shared library is missing the first call raises; there is no
other implementation behind these names.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfrnnt.so")

UNTILED, TILED = 0, 1
F32, BF16 = 0, 1
PATH_AUTO, PATH_SIMT = 0, 1

OK = 0
STATUS_LENGTH, STATUS_LABEL, STATUS_TIMEOUT, STATUS_BOUNDS = 1, 2, 4, 8

EXPORTED = ("frnnt_workspace_size", "frnnt_fwd_bwd", "frnnt_error_string", "frnnt_version", "frnnt_profile",
            "frnnt_profile_read", "frnnt_fwd_bwd_noalloc", "frnnt_fwd_bwd_pruned", "frnnt_fwd_bwd_tdt")
MAX_DURATIONS = 8
NOALLOC_MAX_BYTES = 64 * 1024 * 1024
TEST_HOOKS = ("frnnt_test_gemm_bf16", "frnnt_test_joint_variant", "frnnt_test_lose_gemm_loads")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("U", ctypes.c_int), ("D_enc", ctypes.c_int),
                ("D_pred", ctypes.c_int), ("H", ctypes.c_int), ("V", ctypes.c_int), ("blank", ctypes.c_int),
                ("dtype", ctypes.c_int), ("mode", ctypes.c_int), ("path", ctypes.c_int),
                ("chunk_cells", ctypes.c_int), ("loss", ctypes.c_int), ("prune_S", ctypes.c_int),
                ("n_dur", ctypes.c_int), ("durations", ctypes.c_int * 8), ("wgrad_f32", ctypes.c_int)]


class StageStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int), ("calls", ctypes.c_int),
                ("ms", ctypes.c_double)]


class FrnntError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"frnnt error {code}: {msg}")
        self.code = code


class FrnntStatusError(RuntimeError):
    def __init__(self, bits: int):
        names = [n for n, v in (("invalid lengths", STATUS_LENGTH), ("invalid labels", STATUS_LABEL),
                                ("a bounded device wait timed out", STATUS_TIMEOUT),
                                ("invalid pruning bounds", STATUS_BOUNDS))
                 if bits & v]
        super().__init__(f"frnnt device status {bits}: {'; '.join(names)}")
        self.bits = bits


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded shared library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m rnn_joint_network_02_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32p, f32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        L.frnnt_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(ctypes.c_size_t)]
        L.frnnt_workspace_size.restype = ctypes.c_int
        L.frnnt_fwd_bwd.argtypes = ([ctypes.POINTER(Dims)] + [vp] * 6 + [i32p] * 3 + [f32p, f32p] + [vp] * 6 +
                                    [vp, ctypes.c_size_t, i32p, vp])
        L.frnnt_fwd_bwd.restype = ctypes.c_int
        L.frnnt_fwd_bwd_pruned.argtypes = ([ctypes.POINTER(Dims)] + [vp] * 6 + [i32p] * 4 + [f32p, f32p] + [vp] * 6 +
                                           [vp, ctypes.c_size_t, i32p, vp])
        L.frnnt_fwd_bwd_pruned.restype = ctypes.c_int
        L.frnnt_fwd_bwd_tdt.argtypes = ([ctypes.POINTER(Dims)] + [vp] * 8 + [i32p] * 3 + [f32p, f32p] + [vp] * 8 +
                                        [vp, ctypes.c_size_t, i32p, vp])
        L.frnnt_fwd_bwd_tdt.restype = ctypes.c_int
        L.frnnt_fwd_bwd_noalloc.argtypes = ([ctypes.POINTER(Dims)] + [vp] * 6 + [i32p] * 3 + [f32p, f32p] +
                                            [vp] * 6 + [i32p, vp])
        L.frnnt_fwd_bwd_noalloc.restype = ctypes.c_int
        L.frnnt_error_string.argtypes = [ctypes.c_int]
        L.frnnt_error_string.restype = ctypes.c_char_p
        L.frnnt_version.argtypes = []
        L.frnnt_version.restype = ctypes.c_char_p
        L.frnnt_profile.argtypes = [ctypes.c_int]
        L.frnnt_profile.restype = ctypes.c_int
        L.frnnt_profile_read.argtypes = [ctypes.POINTER(StageStat), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        L.frnnt_profile_read.restype = ctypes.c_int
        L.frnnt_test_gemm_bf16.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int,
                                           ctypes.c_longlong, vp, ctypes.c_int, ctypes.c_longlong, ctypes.c_int,
                                           ctypes.c_int, vp, ctypes.c_longlong, ctypes.c_int, vp, vp]
        L.frnnt_test_gemm_bf16.restype = ctypes.c_int
        L.frnnt_test_joint_variant.argtypes = [ctypes.c_int]
        L.frnnt_test_joint_variant.restype = ctypes.c_int
        L.frnnt_test_lose_gemm_loads.argtypes = [ctypes.c_int]
        L.frnnt_test_lose_gemm_loads.restype = ctypes.c_int
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().frnnt_error_string(code).decode()


def version() -> str:
    return lib().frnnt_version().decode()


def profile(enable: bool) -> None:
    """Per-stage CUDA-event timing on/off for later calls (launch counts are always kept)."""
    lib().frnnt_profile(1 if enable else 0)


def profile_read() -> dict:
    """{stage: dict(launches, calls, ms)} accumulated since the previous read (then reset)."""
    cap = 64
    arr = (StageStat * cap)()
    n = ctypes.c_int(0)
    rc = lib().frnnt_profile_read(arr, cap, ctypes.byref(n))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    out = {}
    for i in range(min(n.value, cap)):
        st = arr[i]
        if st.calls or st.launches:
            out[st.name.decode()] = dict(launches=st.launches, calls=st.calls, ms=st.ms)
    return out


LOSSES = {"marginal": 0, "viterbi": 1}


def make_dims(B, T, U, D_enc, D_pred, H, V, dtype="bf16", mode="tiled", path="auto", chunk_cells=0,
              blank=0, loss="marginal", prune_S=0, durations=(), wgrad_f32=False) -> Dims:
    """``durations`` (token-and-duration transducer): the duration set, or () for the transducer.
    ``wgrad_f32``: weight gradients come back as the library's fp32 accumulators."""
    if len(durations) > MAX_DURATIONS:
        raise ValueError(f"at most {MAX_DURATIONS} durations")
    dur = (ctypes.c_int * 8)(*[int(x) for x in durations])
    return Dims(B, T, U, D_enc, D_pred, H, V, blank, BF16 if dtype == "bf16" else F32,
                TILED if mode == "tiled" else UNTILED, PATH_SIMT if path == "simt" else PATH_AUTO,
                chunk_cells, LOSSES[loss], prune_S, len(durations), dur, 1 if wgrad_f32 else 0)


def workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    rc = lib().frnnt_workspace_size(ctypes.byref(dims), ctypes.byref(n))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    return n.value


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def dims_of(f, g, W_o, dtype, mode, path, chunk_cells, blank, loss="marginal", prune_S=0, durations=(),
            wgrad_f32=False) -> Dims:
    B, T, D_enc = f.shape
    U = g.shape[1] - 1
    V, H = W_o.shape
    return make_dims(B, T, U, D_enc, g.shape[2], H, V, dtype, mode, path, chunk_cells, blank, loss, prune_S,
                     durations, wgrad_f32)


def _check_call(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, out, bounds=None, W_d=None, b_d=None,
                wgrad_f32=False):
    """Host-side checks before any pointer reaches the library: a tensor of the
    wrong shape, dtype, layout or device would otherwise be read or written out
    of bounds by the kernels.  Shapes and dtypes are checked first, then that
    every tensor lives on the same CUDA device.  Raises ValueError."""
    if f.dim() != 3 or g.dim() != 3 or W_o.dim() != 2:
        raise ValueError("f must be [B, T, D_enc], g [B, U+1, D_pred] and W_o [V, H]")
    B, T, D_enc = f.shape
    Up1, D_pred = g.shape[1], g.shape[2]
    V, H = W_o.shape
    ft = f.dtype
    if ft not in (torch.float32, torch.bfloat16):
        raise ValueError(f"f must be float32 or bfloat16, not {ft}")
    want = [("f", f, (B, T, D_enc), ft), ("g", g, (B, Up1, D_pred), ft), ("W_f", W_f, (D_enc, H), ft),
            ("W_g", W_g, (D_pred, H), ft), ("W_o", W_o, (V, H), ft), ("b_o", b_o, (V,), ft),
            ("labels", labels, (B, Up1 - 1), torch.int32), ("T_len", T_len, (B,), torch.int32),
            ("U_len", U_len, (B,), torch.int32)]
    if grad_loss is not None:
        want.append(("grad_loss", grad_loss, (B,), torch.float32))
    if bounds is not None:
        want.append(("bounds", bounds, (B, T), torch.int32))
    if W_d is not None or b_d is not None:
        if W_d is None or b_d is None or W_d.dim() != 2:
            raise ValueError("the duration head needs W_d [n_dur, H] and b_d [n_dur]")
        want += [("W_d", W_d, (W_d.shape[0], H), ft), ("b_d", b_d, (W_d.shape[0],), ft)]
    if out is not None:
        wt = torch.float32 if wgrad_f32 else ft     # dtype of the weight gradients
        want += [("out.loss", out.loss, (B,), torch.float32), ("out.df", out.df, tuple(f.shape), ft),
                 ("out.dg", out.dg, tuple(g.shape), ft), ("out.dW_f", out.dW_f, (D_enc, H), wt),
                 ("out.dW_g", out.dW_g, (D_pred, H), wt), ("out.dW_o", out.dW_o, (V, H), wt),
                 ("out.db_o", out.db_o, (V,), wt), ("out.status", out.status, (4,), torch.int32)]
        if W_d is not None:
            if out.dW_d is None or out.db_d is None:
                raise ValueError("out has no duration-head gradients")
            want += [("out.dW_d", out.dW_d, tuple(W_d.shape), wt), ("out.db_d", out.db_d, tuple(b_d.shape), wt)]
    for name, t, shape, dt in want:
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != dt:
            raise ValueError(f"{name} is {t.dtype}, expected {dt}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if f.device.type != "cuda":
        raise ValueError("the library computes on the GPU: pass CUDA tensors")
    for name, t, _, _ in want:
        if t.device != f.device:
            raise ValueError(f"{name} is on {t.device}, the call's tensors on {f.device}")
    if out is not None and out.workspace is not None and out.workspace.device != f.device:
        raise ValueError(f"the workspace is on {out.workspace.device}, the call's tensors on {f.device}")


class Outputs:
    """Preallocated outputs and workspace of one call shape.

    With ``dims.wgrad_f32`` the weight gradients (dW_f, dW_g, dW_o, db_o and
    the duration head's dW_d, db_d) are fp32 views into one flat buffer,
    ``wflat``, so a data-parallel exchange sums them with one all-reduce."""

    def __init__(self, f, g, W_f, W_g, W_o, b_o, dims: Dims, with_workspace: bool = True, W_d=None, b_d=None):
        dev = f.device
        self.loss = torch.empty(f.shape[0], dtype=torch.float32, device=dev)
        self.df = torch.empty_like(f)
        self.dg = torch.empty_like(g)
        weights = [("dW_f", W_f), ("dW_g", W_g), ("dW_o", W_o), ("db_o", b_o)]
        if W_d is not None:
            weights += [("dW_d", W_d), ("db_d", b_d)]
        self.dW_d = self.db_d = None
        self.wflat = None
        if dims.wgrad_f32:
            # segments start on 16-byte boundaries (the library's alignment rule)
            sizes = [(t.numel() + 3) // 4 * 4 for _, t in weights]
            self.wflat = torch.zeros(sum(sizes), dtype=torch.float32, device=dev)
            off = 0
            for (name, t), n in zip(weights, sizes):
                setattr(self, name, self.wflat[off:off + t.numel()].view(t.shape))
                off += n
        else:
            for name, t in weights:
                setattr(self, name, torch.empty_like(t))
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        n = max(workspace_size(dims), 16) if with_workspace else 16
        self.workspace = torch.empty(n, dtype=torch.uint8, device=dev)

    def grads(self):
        d = dict(df=self.df, dg=self.dg, dW_f=self.dW_f, dW_g=self.dW_g, dW_o=self.dW_o, db_o=self.db_o)
        if self.dW_d is not None:
            d.update(dW_d=self.dW_d, db_d=self.db_d)
        return d


def fwd_bwd(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss=None, mode="tiled", path="auto",
            chunk_cells=0, blank=0, out: Outputs | None = None, check=True, stream=None, loss="marginal",
            wgrad_f32=False):
    """One call of frnnt_fwd_bwd on CUDA tensors.

    Float tensors are all float32 or all bfloat16; labels/T_len/U_len int32.
    ``loss`` is "marginal" (every alignment) or "viterbi" (the best one).
    ``wgrad_f32``: the weight gradients come back in fp32 (unrounded).
    Returns (loss [B] fp32, dict of gradients).  With ``check`` the device
    status word is read back (one 4-byte device-to-host copy, which
    synchronises the stream) and a non-zero status raises FrnntStatusError.
    """
    _check_call(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, out, wgrad_f32=wgrad_f32)
    dtype = "bf16" if f.dtype == torch.bfloat16 else "f32"
    dims = dims_of(f, g, W_o, dtype, mode, path, chunk_cells, blank, loss, wgrad_f32=wgrad_f32)
    if out is None:
        out = Outputs(f, g, W_f, W_g, W_o, b_o, dims)
    if stream is None:
        stream = torch.cuda.current_stream(f.device)
    rc = lib().frnnt_fwd_bwd(ctypes.byref(dims), _ptr(f), _ptr(g), _ptr(W_f), _ptr(W_g), _ptr(W_o), _ptr(b_o),
                             _ptr(labels), _ptr(T_len), _ptr(U_len), _ptr(grad_loss), _ptr(out.loss),
                             _ptr(out.df), _ptr(out.dg), _ptr(out.dW_f), _ptr(out.dW_g), _ptr(out.dW_o),
                             _ptr(out.db_o), _ptr(out.workspace), out.workspace.numel(), _ptr(out.status),
                             ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    if check:
        bits = int(out.status[0].item())
        if bits:
            raise FrnntStatusError(bits)
    return out.loss, out.grads()


def fwd_bwd_noalloc(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss=None, mode="tiled", path="auto",
                    chunk_cells=0, blank=0, out: Outputs | None = None, check=True, stream=None,
                    loss="marginal"):
    """frnnt_fwd_bwd_noalloc: like fwd_bwd, but the library's fixed scratch
    array replaces the workspace (``out.workspace`` is not used).  Raises
    FrnntError(FRNNT_ERR_WORKSPACE) when these dims need more than
    NOALLOC_MAX_BYTES of scratch."""
    _check_call(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, out)
    dtype = "bf16" if f.dtype == torch.bfloat16 else "f32"
    dims = dims_of(f, g, W_o, dtype, mode, path, chunk_cells, blank, loss)
    if out is None:
        out = Outputs(f, g, W_f, W_g, W_o, b_o, dims, with_workspace=False)
    if stream is None:
        stream = torch.cuda.current_stream(f.device)
    rc = lib().frnnt_fwd_bwd_noalloc(ctypes.byref(dims), _ptr(f), _ptr(g), _ptr(W_f), _ptr(W_g), _ptr(W_o),
                                     _ptr(b_o), _ptr(labels), _ptr(T_len), _ptr(U_len), _ptr(grad_loss),
                                     _ptr(out.loss), _ptr(out.df), _ptr(out.dg), _ptr(out.dW_f), _ptr(out.dW_g),
                                     _ptr(out.dW_o), _ptr(out.db_o), _ptr(out.status),
                                     ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        msg = error_string(rc)
        if rc == 3:
            msg += f" (these dims need {workspace_size(dims)} bytes; the fixed scratch holds {NOALLOC_MAX_BYTES})"
        raise FrnntError(rc, msg)
    if check:
        bits = int(out.status[0].item())
        if bits:
            raise FrnntStatusError(bits)
    return out.loss, out.grads()


def test_gemm_bf16(A, B, a_mn: bool, b_mn: bool, M: int, N: int, K: int, epi: int = 0, k_splits: int = 1,
                   out=None, stream=None, variant: int = -1, status=None):
    """Test hook: the tensor-core GEMM D = A * B (see include/frnnt_testing.h).
    A is [M][K] (a_mn False) or [K][M]; B is [N][K] (b_mn False) or [K][N]."""
    if out is None:
        out = torch.zeros(M, N, dtype=torch.bfloat16 if epi in (1, 3) else torch.float32, device=A.device)
    if stream is None:
        stream = torch.cuda.current_stream(A.device)
    rc = lib().frnnt_test_gemm_bf16(M, N, K, _ptr(A), int(a_mn), A.stride(0), _ptr(B), int(b_mn), B.stride(0), epi,
                                    k_splits, _ptr(out), out.stride(0), variant, _ptr(status),
                                    ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    return out


def lose_gemm_loads(n: int) -> int:
    """Test setting (include/frnnt_testing.h): the next n tensor-core GEMM
    launches drop their first K block load, so their bounded wait runs out and
    the status word gets STATUS_TIMEOUT.  Returns the previous count."""
    return int(lib().frnnt_test_lose_gemm_loads(int(n)))


def set_joint_variant(variant: int) -> int:
    """Test hook: fused joint kernel variant for later calls (-1 automatic,
    0 one CTA per cell tile, 1 CTA pairs); returns the previous setting."""
    return int(lib().frnnt_test_joint_variant(int(variant)))


def fwd_bwd_pruned(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, bounds, S: int, grad_loss=None, mode="tiled",
                   path="auto", chunk_cells=0, blank=0, out: Outputs | None = None, check=True, stream=None,
                   loss="marginal", wgrad_f32=False):
    """frnnt_fwd_bwd_pruned: the loss and gradients on the pruned lattice that
    keeps, for frame t of utterance b, the S label positions
    bounds[b,t] <= u < bounds[b,t] + S (bounds: int32 [B, T] on the device)."""
    _check_call(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, out, bounds=bounds, wgrad_f32=wgrad_f32)
    dtype = "bf16" if f.dtype == torch.bfloat16 else "f32"
    dims = dims_of(f, g, W_o, dtype, mode, path, chunk_cells, blank, loss, S, wgrad_f32=wgrad_f32)
    if out is None:
        out = Outputs(f, g, W_f, W_g, W_o, b_o, dims)
    if stream is None:
        stream = torch.cuda.current_stream(f.device)
    rc = lib().frnnt_fwd_bwd_pruned(ctypes.byref(dims), _ptr(f), _ptr(g), _ptr(W_f), _ptr(W_g), _ptr(W_o),
                                    _ptr(b_o), _ptr(labels), _ptr(T_len), _ptr(U_len), _ptr(bounds),
                                    _ptr(grad_loss), _ptr(out.loss), _ptr(out.df), _ptr(out.dg), _ptr(out.dW_f),
                                    _ptr(out.dW_g), _ptr(out.dW_o), _ptr(out.db_o), _ptr(out.workspace),
                                    out.workspace.numel(), _ptr(out.status), ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    if check:
        bits = int(out.status[0].item())
        if bits:
            raise FrnntStatusError(bits)
    return out.loss, out.grads()


def fwd_bwd_tdt(f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, durations, grad_loss=None,
                mode="tiled", chunk_cells=0, blank=0, out: Outputs | None = None, check=True, stream=None,
                wgrad_f32=False):
    """frnnt_fwd_bwd_tdt: the token-and-duration transducer loss and gradients.

    W_d [n_dur, H] and b_d [n_dur] are the duration head (bf16, like the other
    weights); ``durations`` is the duration set (frame counts, increasing,
    starting 0, 1).  Returns (loss [B] fp32, dict of gradients including dW_d
    and db_d)."""
    _check_call(f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, out, W_d=W_d, b_d=b_d,
                wgrad_f32=wgrad_f32)
    dtype = "bf16" if f.dtype == torch.bfloat16 else "f32"
    dims = dims_of(f, g, W_o, dtype, mode, "auto", chunk_cells, blank, "marginal", 0, tuple(durations),
                   wgrad_f32=wgrad_f32)
    if out is None:
        out = Outputs(f, g, W_f, W_g, W_o, b_o, dims, W_d=W_d, b_d=b_d)
    if stream is None:
        stream = torch.cuda.current_stream(f.device)
    rc = lib().frnnt_fwd_bwd_tdt(ctypes.byref(dims), _ptr(f), _ptr(g), _ptr(W_f), _ptr(W_g), _ptr(W_o), _ptr(b_o),
                                 _ptr(W_d), _ptr(b_d), _ptr(labels), _ptr(T_len), _ptr(U_len), _ptr(grad_loss),
                                 _ptr(out.loss), _ptr(out.df), _ptr(out.dg), _ptr(out.dW_f), _ptr(out.dW_g),
                                 _ptr(out.dW_o), _ptr(out.db_o), _ptr(out.dW_d), _ptr(out.db_d),
                                 _ptr(out.workspace), out.workspace.numel(), _ptr(out.status),
                                 ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        raise FrnntError(rc, error_string(rc))
    if check:
        bits = int(out.status[0].item())
        if bits:
            raise FrnntStatusError(bits)
    return out.loss, out.grads()
