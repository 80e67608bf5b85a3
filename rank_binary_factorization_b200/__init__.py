"""B200 (sm_100a) NanoQuant hot path: calibration preconditioners and LB-ADMM.

Thin torch-facing binding of the C ABI in ``include/nq.h``.  Every function here only
marshals arguments (torch tensors for device memory, torch's current CUDA stream) and
calls the library of the same name; all computation runs in the CUDA kernels of
``libnq.so``.  Importing this package without the built library raises ImportError.
"""
import ctypes
import os

import torch

from . import build as _build

if os.environ.get("NQ_NO_AUTOBUILD") != "1":
    _build.build()          # no-op unless libnq.so is missing or older than its sources

from . import _lib
from ._lib import (FIELDS, NQ_BF16, NQ_F32, NQ_PREC_BF16, NQ_PREC_FP32, NQError, check, lib,
                   status_string)

__all__ = [
    "nq_bpw", "nq_rank_for_bpw", "nq_calib_stats", "nq_calib_precond", "nq_lbadmm",
    "nq_recon_error", "nq_pack_signs", "nq_binary_matmul", "nq_ls_refit", "LBState", "NQError",
    "status_string", "lib",
    "nq_launch_count", "nq_profile_enable", "nq_profile_get", "nq_selftest",
    "nq_set_inverse_mode", "nq_set_tuning", "nq_set_latent_solver",
]


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return NQ_BF16
    if t.dtype == torch.float32:
        return NQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


def _cuda(t, name):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t


def workspace(nbytes, device=None):
    """A 256-byte aligned device buffer (torch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")


def nq_bpw(m, n, r):
    return lib.nq_bpw(m, n, r)


def nq_rank_for_bpw(m, n, bpw):
    return lib.nq_rank_for_bpw(m, n, float(bpw))


def nq_calib_stats(X, ws=None):
    """(s, q) float64 per-channel mean x^2 and mean x^4 of a T x C stream."""
    _cuda(X, "X")
    T, C = X.shape
    ws = ws if ws is not None else workspace(lib.nq_calib_workspace_size(T, C), X.device)
    s = torch.empty(C, dtype=torch.float64, device=X.device)
    q = torch.empty(C, dtype=torch.float64, device=X.device)
    check("nq_calib_stats", lib.nq_calib_stats(_ptr(X), T, C, _dtype(X), _ptr(s), _ptr(q),
                                               _ptr(ws), ws.numel(), _stream()))
    return s, q


def nq_calib_precond(acts, grads, alpha_override=-1.0, ws=None, sync=True):
    """(d_in, d_out, alpha_in, alpha_out) from activation (T_in x n) and gradient (T_out x m) streams."""
    _cuda(acts, "acts")
    _cuda(grads, "grads")
    if acts.dtype != grads.dtype:
        raise TypeError("acts and grads must share a dtype")
    T_in, n = acts.shape
    T_out, m = grads.shape
    need = lib.nq_calib_workspace_size(max(T_in, T_out), max(n, m))
    ws = ws if ws is not None else workspace(need, acts.device)
    d_in = torch.empty(n, dtype=torch.float32, device=acts.device)
    d_out = torch.empty(m, dtype=torch.float32, device=acts.device)
    alpha = (ctypes.c_double * 2)() if sync else None
    check("nq_calib_precond", lib.nq_calib_precond(
        _ptr(acts), T_in, n, _ptr(grads), T_out, m, _dtype(acts), float(alpha_override),
        _ptr(d_in), _ptr(d_out), alpha if sync else None, _ptr(ws), ws.numel(), _stream()))
    if sync:
        return d_in, d_out, alpha[0], alpha[1]
    return d_in, d_out, None, None


def nq_lbadmm(W, r, d_in=None, d_out=None, rho=1.0, lam=1e-4, iters=30, K=4, seed=0, ws=None,
              want_objective=True, want_error=True):
    """Full LB-ADMM on one layer.

    Returns dict(U_packed, V_packed, s1, s2, objective (list or None), rel_err (float or None)).
    """
    _cuda(W, "W")
    m, n = W.shape
    dev = W.device
    ws = ws if ws is not None else workspace(lib.nq_lbadmm_workspace_size(m, n, r), dev)
    nw = (r + 31) // 32
    Up = torch.empty(m, nw, dtype=torch.int32, device=dev)
    Vp = torch.empty(n, nw, dtype=torch.int32, device=dev)
    s1 = torch.empty(m, dtype=torch.float32, device=dev)
    s2 = torch.empty(n, dtype=torch.float32, device=dev)
    obj = (ctypes.c_float * iters)() if want_objective else None
    err = ctypes.c_float(0.0)
    check("nq_lbadmm", lib.nq_lbadmm(
        _ptr(W), _dtype(W), m, n, _ptr(d_in), _ptr(d_out), r, rho, lam, iters, K, seed, _ptr(Up),
        _ptr(Vp), _ptr(s1), _ptr(s2), obj, ctypes.byref(err) if want_error else None, _ptr(ws),
        ws.numel(), _stream()))
    return dict(U_packed=Up, V_packed=Vp, s1=s1, s2=s2,
                objective=list(obj) if want_objective else None,
                rel_err=err.value if want_error else None)


def nq_recon_error(W, U_packed, V_packed, r, s1, s2, d_in=None, d_out=None, ws=None):
    _cuda(W, "W")
    m, n = W.shape
    ws = ws if ws is not None else workspace(lib.nq_recon_workspace_size(m, n, r), W.device)
    out = ctypes.c_double(0.0)
    check("nq_recon_error", lib.nq_recon_error(
        _ptr(W), _dtype(W), m, n, _ptr(d_in), _ptr(d_out), _ptr(U_packed), _ptr(V_packed), r,
        _ptr(s1), _ptr(s2), ctypes.byref(out), _ptr(ws), ws.numel(), _stream()))
    return out.value


def nq_binary_matmul(U_packed, V_packed, s1, s2, r, X, ws=None):
    """Y = X diag(s2) V+- U+-^T diag(s1) for X of shape (B, n) or (n,); returns float32 Y."""
    _cuda(X, "X")
    vec = X.dim() == 1
    X2 = X.unsqueeze(0) if vec else X
    B, n = X2.shape
    m = s1.shape[0]
    need = lib.nq_binary_workspace_size(m, n, r, B)
    ws = ws if ws is not None else workspace(need, X.device)
    Y = torch.empty(B, m, dtype=torch.float32, device=X.device)
    check("nq_binary_matmul", lib.nq_binary_matmul(
        _ptr(U_packed), _ptr(V_packed), _ptr(s1), _ptr(s2), m, n, r, _ptr(X2), _dtype(X2), B,
        _ptr(Y), _ptr(ws), ws.numel(), _stream()))
    return Y[0] if vec else Y


def nq_ls_refit(W, U_packed, V_packed, r, s1, s2, d_in=None, d_out=None, sweeps=3, ws=None,
                want_error=True):
    """Least-squares refit of s1, s2 (updated in place) for the fixed packed signs; returns
    the reconstruction error after the refit (or None)."""
    _cuda(W, "W")
    m, n = W.shape
    ws = ws if ws is not None else workspace(lib.nq_ls_refit_workspace_size(m, n, r), W.device)
    out = ctypes.c_double(0.0)
    check("nq_ls_refit", lib.nq_ls_refit(
        _ptr(W), _dtype(W), m, n, _ptr(d_in), _ptr(d_out), _ptr(U_packed), _ptr(V_packed), r,
        _ptr(s1), _ptr(s2), sweeps, ctypes.byref(out) if want_error else None, _ptr(ws),
        ws.numel(), _stream()))
    return out.value if want_error else None


def nq_pack_signs(X):
    _cuda(X, "X")
    rows, r = X.shape
    bits = torch.empty(rows, (r + 31) // 32, dtype=torch.int32, device=X.device)
    check("nq_pack_signs", lib.nq_pack_signs(_ptr(X), rows, r, _ptr(bits), _stream()))
    return bits


def nq_set_inverse_mode(mode):
    """How each half step forms G^-1: "auto", "cholesky" or "newton" (process-wide)."""
    code = {"auto": _lib.NQ_INV_AUTO, "cholesky": _lib.NQ_INV_CHOLESKY,
            "newton": _lib.NQ_INV_NEWTON}[mode]
    check("nq_set_inverse_mode", lib.nq_set_inverse_mode(code))


def nq_set_latent_solver(solver="exact", gd_steps=8):
    """Latent update of each half step: "exact" (default) or "gd" (gd_steps gradient steps)."""
    code = {"exact": _lib.NQ_SOLVER_EXACT, "gd": _lib.NQ_SOLVER_GD}[solver]
    check("nq_set_latent_solver", lib.nq_set_latent_solver(code, int(gd_steps)))


def nq_set_tuning(key, value):
    """Scheduling setting ("factor_ctas", "newton_bn", "svid_beside", "nfast", "rhs_bn",
    "solve_bn", "newton_fused"; see nq_tuning)."""
    check("nq_set_tuning", lib.nq_set_tuning(_lib.TUNING[key], int(value)))


def nq_launch_count():
    """Kernel launches issued by the library so far in this process."""
    return lib.nq_launch_count()


def nq_profile_enable(on=True):
    check("nq_profile_enable", lib.nq_profile_enable(1 if on else 0))


def nq_profile_get():
    """{kernel class: (launch scopes, device ms)} recorded since nq_profile_enable(True)."""
    out = {}
    for i, name in enumerate(_lib.KERNEL_CLASSES):
        n, ms = ctypes.c_int64(), ctypes.c_double()
        check("nq_profile_get", lib.nq_profile_get(i, ctypes.byref(n), ctypes.byref(ms)))
        out[name] = (n.value, ms.value)
    return out


def nq_selftest(kind):
    """Run a device-side error path on purpose ("wait_timeout" or "not_spd"); returns the
    status code the library reports (NQ_ERR_TIMEOUT / NQ_ERR_NOT_SPD expected)."""
    code = {"wait_timeout": _lib.NQ_SELFTEST_WAIT_TIMEOUT,
            "not_spd": _lib.NQ_SELFTEST_NOT_SPD}[kind]
    ws = workspace(lib.nq_selftest_workspace_size())
    return lib.nq_selftest(code, _ptr(ws), ws.numel(), _stream())


class LBState:
    """Step-level access to an LB-ADMM workspace (prepare / half steps / state fields).

    ``prec`` is the operand precision of the contractions ("bf16" or "fp32", see
    nq_precision); nq_lbadmm picks "fp32" for FP32 weights and "bf16" for BF16 weights.
    """

    _DT = {2: torch.bfloat16, 4: torch.float32, 8: torch.float64}

    def __init__(self, m, n, r, device="cuda", prec="bf16"):
        self.m, self.n, self.r = m, n, r
        self.prec = {"bf16": NQ_PREC_BF16, "fp32": NQ_PREC_FP32}[prec]
        self.nbytes = lib.nq_lbadmm_workspace_size(m, n, r)
        if self.nbytes == 0:
            raise NQError("nq_lbadmm_workspace_size", _lib.NQ_ERR_INVALID_ARG)
        self.ws = workspace(self.nbytes, device)

    def _args(self):
        return self.m, self.n, self.r

    def prepare(self, W, d_in=None, d_out=None, seed=0):
        g = ctypes.c_double(0.0)
        check("nq_lbadmm_prepare", lib.nq_lbadmm_prepare(
            _ptr(W), _dtype(W), self.m, self.n, _ptr(d_in), _ptr(d_out), self.r, seed,
            self.prec, ctypes.byref(g), _ptr(self.ws), self.nbytes, _stream()))
        return g.value

    def iterate(self, iters, rho=1.0, lam=1e-4, K=4, want_objective=True):
        obj = (ctypes.c_float * iters)() if want_objective else None
        check("nq_lbadmm_iterate", lib.nq_lbadmm_iterate(
            *self._args(), rho, lam, iters, K, self.prec, obj, _ptr(self.ws), self.nbytes,
            _stream()))
        return list(obj) if want_objective else None

    def half_step(self, side, rho=1.0, lam=1e-4, K=4):
        check("nq_lbadmm_half_step", lib.nq_lbadmm_half_step(
            *self._args(), rho, lam, K, side, self.prec, _ptr(self.ws), self.nbytes, _stream()))

    def finish(self, W=None, d_in=None, d_out=None, want_error=True):
        m, n, r = self._args()
        dev = self.ws.device
        nw = (r + 31) // 32
        Up = torch.empty(m, nw, dtype=torch.int32, device=dev)
        Vp = torch.empty(n, nw, dtype=torch.int32, device=dev)
        s1 = torch.empty(m, dtype=torch.float32, device=dev)
        s2 = torch.empty(n, dtype=torch.float32, device=dev)
        err = ctypes.c_float(0.0)
        check("nq_lbadmm_finish", lib.nq_lbadmm_finish(
            _ptr(W), _dtype(W) if W is not None else NQ_F32, m, n, _ptr(d_in), _ptr(d_out), r,
            _ptr(Up), _ptr(Vp), _ptr(s1), _ptr(s2), ctypes.byref(err) if want_error else None,
            _ptr(self.ws), self.nbytes, _stream()))
        return dict(U_packed=Up, V_packed=Vp, s1=s1, s2=s2,
                    rel_err=err.value if want_error else None)

    def field(self, name):
        """A torch view (rows x ld, or flat) of one state field inside the workspace."""
        ptr, cnt, eb, ld = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int64()
        check("nq_lbadmm_state_field", lib.nq_lbadmm_state_field(
            *self._args(), FIELDS[name], _ptr(self.ws), self.nbytes, ctypes.byref(ptr),
            ctypes.byref(cnt), ctypes.byref(eb), ctypes.byref(ld)))
        off = ptr.value - self.ws.data_ptr()
        flat = self.ws[off:off + cnt.value * eb.value].view(self._DT[eb.value])
        if ld.value > 1:
            return flat.view(-1, ld.value)
        return flat

    def inv_stats(self):
        """Counters of the Newton-Schulz inverse update: accepted half steps, fallbacks to
        Cholesky, steps of the last accepted update, ||I - X_k G||_F of the last attempt."""
        w = self.field("INV_STATS").cpu()
        i = w.view(torch.int64)
        return dict(accepted=int(i[0]), fallbacks=int(i[1]), steps=int(i[2]),
                    residuals=[float(x) for x in w[3:]])

    def ginv(self, side):
        """G^-1 (hi + lo, FP32, r x r) of the last solve of ``side`` (0: U, 1: V)."""
        nm = "GINV_U" if side == 0 else "GINV_V"
        r = self.r
        return self.field(nm)[:r, :r].float() + self.field(nm + "_LO")[:r, :r].float()

    def sync_operands(self):
        check("nq_lbadmm_sync_operands", lib.nq_lbadmm_sync_operands(
            *self._args(), self.prec, _ptr(self.ws), self.nbytes, _stream()))

    def check_device_error(self):
        return lib.nq_lbadmm_check(*self._args(), _ptr(self.ws), self.nbytes, _stream())
