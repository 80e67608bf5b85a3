"""Host-side checks of the C ABI (CPU only: no kernel is launched).

The library must load, export every function that include/nq.h declares, compute
the BPW helpers exactly like the oracle's closed forms, and reject bad arguments
before it touches a device.
"""
import ctypes
import os
import re
from fractions import Fraction

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    import rank_binary_factorization_b200 as nq
    return nq


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "nq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound():
    nq = _lib()
    names = _declared_functions()
    assert len(names) >= 19
    for name in names:
        assert hasattr(nq.lib, name), name
    from rank_binary_factorization_b200._lib import SIGNATURES
    assert set(SIGNATURES) == set(names)


def test_version_and_status_strings():
    nq = _lib()
    assert nq.lib.nq_version() == 100
    assert nq.status_string(0) == "NQ_OK"
    assert nq.status_string(5) == "NQ_ERR_NOT_SPD"
    assert nq.status_string(99) == "NQ_ERR_UNKNOWN"


@pytest.mark.parametrize("m,n,target", [(4096, 4096, 1.0), (4096, 4096, 0.8), (11008, 4096, 0.8),
                                        (4096, 11008, 0.8), (8192, 8192, 0.55), (1024, 8192, 0.55),
                                        (28672, 8192, 0.55), (8192, 28672, 0.55), (8192, 8192, 1.0),
                                        (256, 512, 0.1875), (17, 33, 3.0), (4, 4, 1.0),
                                        (100, 300, 0.37), (65536, 65536, 2.0)])
def test_bpw_helpers_match_oracle(m, n, target):
    from oracle.bpw import bpw, rank_for_bpw
    nq = _lib()
    r = nq.nq_rank_for_bpw(m, n, target)
    assert r == rank_for_bpw(m, n, target)
    assert abs(nq.nq_bpw(m, n, r) - float(bpw(m, n, r))) < 1e-15


def test_bpw_helpers_reject_bad_sizes():
    nq = _lib()
    assert nq.nq_bpw(0, 4, 1) == -1.0
    assert nq.nq_rank_for_bpw(4, -1, 1.0) == -1
    assert nq.nq_rank_for_bpw(4, 4, -0.5) == -1


def test_workspace_sizes():
    nq = _lib()
    L = nq.lib
    assert L.nq_lbadmm_workspace_size(4096, 4096, 2032) > 4096 * 4096 * 4
    assert L.nq_lbadmm_workspace_size(16, 16, 17) == 0          # r > min(m, n)
    assert L.nq_lbadmm_workspace_size(8192, 8192, 4097) == 0    # r above the supported maximum
    assert L.nq_lbadmm_workspace_size(0, 16, 1) == 0
    assert L.nq_calib_workspace_size(262144, 4096) > 0
    assert L.nq_calib_workspace_size(0, 4096) == 0
    assert L.nq_recon_workspace_size(64, 64, 8) > 0


def test_argument_errors_are_reported_before_any_device_work():
    nq = _lib()
    L = nq.lib
    INV, WS = nq._lib.NQ_ERR_INVALID_ARG, nq._lib.NQ_ERR_WORKSPACE
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced: every call below fails validation first
    # null weight, bad dtype, non-positive rho, zero iterations, K = 0
    assert L.nq_lbadmm(null, 0, 8, 8, null, null, 2, 1.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm(fake, 7, 8, 8, null, null, 2, 1.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm(fake, 0, 8, 8, null, null, 2, 0.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm(fake, 0, 8, 8, null, null, 2, 1.0, 1e-4, 0, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm(fake, 0, 8, 8, null, null, 2, 1.0, 1e-4, 1, 0, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    # diagnostics: unknown kind, null / misaligned / short workspace
    assert L.nq_selftest(7, fake, 1 << 30, null) == INV
    assert L.nq_selftest(0, null, 1 << 30, null) == INV
    assert L.nq_selftest(1, ctypes.c_void_p((1 << 40) + 8), 1 << 30, null) == INV
    assert L.nq_selftest(0, fake, 16, null) == WS
    assert L.nq_selftest_workspace_size() > 64 * 64 * 4
    # rank above min(m, n)
    assert L.nq_lbadmm(fake, 0, 8, 4, null, null, 5, 1.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 1 << 30, null) == INV
    # workspace: misaligned, then too small
    assert L.nq_lbadmm(fake, 0, 8, 8, null, null, 2, 1.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, ctypes.c_void_p((1 << 40) + 8), 1 << 30, null) == INV
    assert L.nq_lbadmm(fake, 0, 8, 8, null, null, 2, 1.0, 1e-4, 1, 1, 0, fake, fake, fake, fake,
                       null, null, fake, 64, null) == WS
    # calibration: empty stream, NaN override, alpha override above 1
    assert L.nq_calib_precond(fake, 0, 4, fake, 4, 4, 1, -1.0, fake, fake, null, fake, 1 << 30,
                              null) == INV
    assert L.nq_calib_precond(fake, 4, 4, fake, 4, 4, 1, float("nan"), fake, fake, null, fake,
                              1 << 30, null) == INV
    assert L.nq_calib_precond(fake, 4, 4, fake, 4, 4, 1, 1.5, fake, fake, null, fake, 1 << 30,
                              null) == INV
    assert L.nq_calib_stats(fake, 4, 4, 1, fake, fake, fake, 16, null) == WS
    # state fields and half steps
    p, c, e, ld = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int64()
    assert L.nq_lbadmm_state_field(8, 8, 2, 42, fake, 1 << 30, ctypes.byref(p), ctypes.byref(c),
                                   ctypes.byref(e), ctypes.byref(ld)) == INV
    assert L.nq_lbadmm_half_step(8, 8, 2, 1.0, 1e-4, 4, 2, 0, fake, 1 << 30, null) == INV
    # unknown precision mode
    assert L.nq_lbadmm_half_step(8, 8, 2, 1.0, 1e-4, 4, 0, 2, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm_iterate(8, 8, 2, 1.0, 1e-4, 1, 4, 9, null, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm_sync_operands(8, 8, 2, -1, fake, 1 << 30, null) == INV
    assert L.nq_lbadmm_prepare(fake, 0, 8, 8, null, null, 2, 0, 3, null, fake, 1 << 30,
                               null) == INV
    assert L.nq_pack_signs(null, 4, 4, fake, null) == INV
    # refit: zero sweeps, null scales; binary matmul: empty batch, null input
    assert L.nq_ls_refit(fake, 0, 8, 8, null, null, fake, fake, 2, fake, fake, 0, null, fake,
                         1 << 30, null) == INV
    assert L.nq_ls_refit(fake, 0, 8, 8, null, null, fake, fake, 2, null, fake, 1, null, fake,
                         1 << 30, null) == INV
    assert L.nq_binary_matmul(fake, fake, fake, fake, 8, 8, 2, fake, 0, 0, fake, fake, 1 << 30,
                              null) == INV
    assert L.nq_binary_matmul(fake, fake, fake, fake, 8, 8, 2, null, 0, 1, fake, fake, 1 << 30,
                              null) == INV


@pytest.mark.parametrize("m,n,r", [(300, 200, 40), (256, 512, 16), (4096, 4096, 2032),
                                   (11008, 4096, 1000), (8192, 8192, 4080), (1024, 8192, 484),
                                   (28672, 8192, 3488), (7, 9, 1)])
def test_state_field_offsets_are_inside_the_workspace(m, n, r):
    nq = _lib()
    L = nq.lib
    size = L.nq_lbadmm_workspace_size(m, n, r)
    base = 1 << 40
    seen = []
    for name, f in nq._lib.FIELDS.items():
        p, c, e, ld = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int64()
        assert L.nq_lbadmm_state_field(m, n, r, f, ctypes.c_void_p(base), size, ctypes.byref(p),
                                       ctypes.byref(c), ctypes.byref(e), ctypes.byref(ld)) == 0
        start, end = p.value - base, p.value - base + c.value * e.value
        assert 0 <= start and end <= size, name
        assert start % (8 if name == "GAMMA" else 256) == 0, name   # regions are 256-aligned
        seen.append((start, end, name))
    seen.sort()
    for (s0, e0, n0), (s1, e1, n1) in zip(seen, seen[1:]):
        assert e0 <= s1, (n0, n1)     # fields do not overlap


def test_inverse_mode_and_tuning_settings_are_checked():
    nq = _lib()
    L = nq.lib
    INV = 1
    for mode in (0, 1, 2):
        assert L.nq_set_inverse_mode(mode) == 0
    assert L.nq_set_inverse_mode(3) == INV and L.nq_set_inverse_mode(-1) == INV
    T = nq._lib.TUNING
    for key, good, bad in (("factor_ctas", (-1, 0, 3, 74, 1000), (-2,)),
                           ("newton_bn", (0, 64, 128, 256), (32, 96, 512, -1)),
                           ("svid_beside", (0, 1), (2, -1)),
                           ("nfast", (0, 1), (2, -1)),
                           ("rhs_bn", (0, 128, 256), (64, 1)),
                           ("solve_bn", (0, 128, 256), (64, 1)),
                           ("newton_fused", (0, 1), (2, -1))):
        for v in good:
            assert L.nq_set_tuning(T[key], v) == 0, (key, v)
        for v in bad:
            assert L.nq_set_tuning(T[key], v) == INV, (key, v)
    assert L.nq_set_tuning(7, 0) == INV
    # back to the defaults
    assert L.nq_set_inverse_mode(0) == 0
    for key, v in (("factor_ctas", -1), ("newton_bn", 0), ("svid_beside", 1), ("nfast", 1),
                   ("rhs_bn", 0), ("solve_bn", 0), ("newton_fused", 0)):
        assert L.nq_set_tuning(T[key], v) == 0


def test_latent_solver_setting_is_checked():
    nq = _lib()
    L = nq.lib
    INV = 1
    assert L.nq_set_latent_solver(1, 8) == 0
    assert L.nq_set_latent_solver(1, 0) == INV and L.nq_set_latent_solver(1, 1001) == INV
    assert L.nq_set_latent_solver(2, 8) == INV and L.nq_set_latent_solver(-1, 8) == INV
    assert L.nq_set_latent_solver(0, 0) == 0      # the step count only matters for GD


def _declared_arities():
    src = open(os.path.join(ROOT, "include", "nq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(nq_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    from rank_binary_factorization_b200._lib import SIGNATURES
    arity = _declared_arities()
    assert set(arity) == set(SIGNATURES)
    for name, (_, args) in SIGNATURES.items():
        assert len(args) == arity[name], (name, len(args), arity[name])
