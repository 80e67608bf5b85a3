"""ctypes binding of ``libnq.so`` (the C ABI declared in include/nq.h).

Argument marshalling only: every step of the computation runs in the CUDA library.
Tensors are passed by ``data_ptr()``; the stream is torch's current CUDA stream.
If the shared library is missing this module raises at import: there is no CPU
fallback.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python rank_binary_factorization_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

c_i32, c_i64, c_u64, c_f32, c_f64 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                      ctypes.c_float, ctypes.c_double)
c_vp, c_sz = ctypes.c_void_p, ctypes.c_size_t

NQ_OK, NQ_ERR_INVALID_ARG, NQ_ERR_WORKSPACE, NQ_ERR_CUDA, NQ_ERR_NONFINITE, NQ_ERR_NOT_SPD, \
    NQ_ERR_TIMEOUT, NQ_ERR_UNSUPPORTED = range(8)
NQ_F32, NQ_BF16 = 0, 1
NQ_PREC_BF16, NQ_PREC_FP32 = 0, 1
FIELDS = dict(U=0, V=1, SU=2, SV=3, AU=4, AV=5, BU=6, BV=7, WHAT=8, GAMMA=9, WHAT_LO=10,
              INV_STATS=11, GINV_U=12, GINV_U_LO=13, GINV_V=14, GINV_V_LO=15)
NQ_INV_AUTO, NQ_INV_CHOLESKY, NQ_INV_NEWTON = 0, 1, 2
NQ_SOLVER_EXACT, NQ_SOLVER_GD = 0, 1
TUNING = dict(factor_ctas=0, newton_bn=1, svid_beside=2, nfast=3, rhs_bn=4, solve_bn=5,
              newton_fused=6)

# name -> (restype, argtypes); the list is the full set of exported entry points
SIGNATURES = {
    "nq_status_string": (ctypes.c_char_p, [c_i32]),
    "nq_version": (c_i32, []),
    "nq_bpw": (c_f64, [c_i64, c_i64, c_i32]),
    "nq_rank_for_bpw": (c_i32, [c_i64, c_i64, c_f64]),
    "nq_calib_workspace_size": (c_sz, [c_i64, c_i64]),
    "nq_calib_stats": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "nq_calib_stats_noalloc": (c_i32, [c_vp, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp]),
    "nq_calib_precond": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_i64, c_i64, c_i32, c_f64, c_vp,
                                 c_vp, c_vp, c_vp, c_sz, c_vp]),
    "nq_lbadmm_workspace_size": (c_sz, [c_i64, c_i64, c_i32]),
    "nq_set_inverse_mode": (c_i32, [c_i32]),
    "nq_set_tuning": (c_i32, [c_i32, c_i32]),
    "nq_set_latent_solver": (c_i32, [c_i32, c_i32]),
    "nq_lbadmm": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_i32, c_f32, c_f32, c_i32,
                          c_i32, c_u64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "nq_recon_workspace_size": (c_sz, [c_i64, c_i64, c_i32]),
    "nq_recon_error": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp,
                               c_vp, c_vp, c_vp, c_sz, c_vp]),
    "nq_pack_signs": (c_i32, [c_vp, c_i64, c_i32, c_vp, c_vp]),
    "nq_binary_workspace_size": (c_sz, [c_i64, c_i64, c_i32, c_i64]),
    "nq_ls_refit_workspace_size": (c_sz, [c_i64, c_i64, c_i32]),
    "nq_ls_refit": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp,
                            c_i32, c_vp, c_vp, c_sz, c_vp]),
    "nq_binary_matmul": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i32, c_vp, c_i32, c_i64,
                                 c_vp, c_vp, c_sz, c_vp]),
    "nq_lbadmm_prepare": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_i32, c_u64, c_i32,
                                  c_vp, c_vp, c_sz, c_vp]),
    "nq_lbadmm_iterate": (c_i32, [c_i64, c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_i32, c_vp,
                                  c_vp, c_sz, c_vp]),
    "nq_lbadmm_half_step": (c_i32, [c_i64, c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_i32, c_vp,
                                    c_sz, c_vp]),
    "nq_lbadmm_finish": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp,
                                 c_vp, c_vp, c_vp, c_sz, c_vp]),
    "nq_lbadmm_state_field": (c_i32, [c_i64, c_i64, c_i32, c_i32, c_vp, c_sz,
                                      ctypes.POINTER(c_vp), ctypes.POINTER(c_i64),
                                      ctypes.POINTER(c_i32), ctypes.POINTER(c_i64)]),
    "nq_lbadmm_sync_operands": (c_i32, [c_i64, c_i64, c_i32, c_i32, c_vp, c_sz, c_vp]),
    "nq_lbadmm_check": (c_i32, [c_i64, c_i64, c_i32, c_vp, c_sz, c_vp]),
    "nq_launch_count": (c_i64, []),
    "nq_profile_enable": (c_i32, [c_i32]),
    "nq_profile_get": (c_i32, [c_i32, ctypes.POINTER(c_i64), ctypes.POINTER(c_f64)]),
    "nq_selftest_workspace_size": (c_sz, []),
    "nq_selftest": (c_i32, [c_i32, c_vp, c_sz, c_vp]),
}
NQ_SELFTEST_WAIT_TIMEOUT, NQ_SELFTEST_NOT_SPD = 0, 1
KERNEL_CLASSES = ["calib", "calib_finalize", "prep", "gram", "chol", "rhs", "solve", "svid",
                  "objective", "finish", "recon", "ginv", "binary", "refit", "newton", "gd"]

for _name, (_res, _args) in SIGNATURES.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class NQError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def status_string(code):
    return lib.nq_status_string(int(code)).decode()


def check(fn, code):
    if code != NQ_OK:
        raise NQError(fn, code)
    return code
