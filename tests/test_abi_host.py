"""Host-side checks of the C ABI: the library loads, exports every function
the header declares, struct layouts agree, and argument errors come back
synchronously before anything is launched (no GPU needed)."""
import ctypes
import os
import re

import pytest

import dimuon_optimizer_b200 as dm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dimuon.h")


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\S.*?\b(dm_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 7
    lib = ctypes.CDLL(dm.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(dm.EXPORTED)


def test_struct_layouts():
    assert ctypes.sizeof(dm.dm_matrix_t) == 80
    assert ctypes.sizeof(dm.dm_hparams_t) == 72
    assert dm.dm_matrix_t.update_out.offset == 72
    assert dm.dm_hparams_t.debug_flags.offset == 44
    assert dm.dm_hparams_t.nesterov.offset == 48
    assert dm.dm_hparams_t.ns_coeffs.offset == 64


def test_defaults_and_strings():
    hp = dm.dm_default_hparams()
    assert (round(hp.a, 4), round(hp.b, 4), round(hp.c, 4)) == (3.4445, -4.775, 2.0315)
    assert hp.ns_steps == 5 and abs(hp.mu - 0.95) < 1e-7 and abs(hp.cond_eps - 1e-4) < 1e-10
    assert hp.precision == dm.DM_PREC_BF16_TC
    assert dm.dm_status_string(dm.DM_OK) == "ok"
    assert "workspace" in dm.dm_status_string(dm.DM_ERR_WORKSPACE)
    assert dm.dm_status_string(1234) == "unknown status"
    assert re.match(r"\d+\.\d+\.\d+", dm.dm_version())


def fake_matrix(rows, cols, wdt=dm.DM_BF16, energies=True):
    m = dm.dm_matrix_t()
    m.rows, m.cols = rows, cols
    m.weight, m.grad, m.momentum = 0x1000, 0x2000, 0x3000
    m.weight_dtype = m.grad_dtype = m.momentum_dtype = wdt
    if energies:
        m.row_energy, m.col_energy = 0x4000, 0x5000
    return m


def test_workspace_size_host_only():
    hp = dm.dm_default_hparams()
    thin = dm.dm_workspace_size([fake_matrix(8, 4096)], hp, 1)
    big = dm.dm_workspace_size([fake_matrix(1024, 1024)], hp, 0)
    big_cond = dm.dm_workspace_size([fake_matrix(1024, 1024)], hp, 1)
    # thin factors: fp64 Gram partials (S_1, S_2) of the four 1024-column slabs
    # of an 8 x 4096 factor (one 8x8 block each), plus small per-factor slots
    assert 1024 + 4 * 2 * 64 * 8 <= thin <= 16 * 1024
    thin32 = dm.dm_workspace_size([fake_matrix(4096, 32)] * 448, hp, 1)
    assert thin32 <= dm.DM_NOALLOC_MAX_BYTES  # a LoRA r=32 set fits the static scratch
    assert big >= 2 * 1024 * 1024 * 2 + 2 * 1024 * 1024 * 2   # X ping-pong + A + B
    assert big_cond > big
    hp32 = dm.dm_default_hparams(precision=dm.DM_PREC_FP32)
    assert dm.dm_workspace_size([fake_matrix(1024, 1024)], hp32, 0) > big
    # the thin threshold can be lifted for testing
    hp_nt = dm.dm_default_hparams(debug_flags=dm.DM_DBG_NO_THIN)
    assert dm.dm_workspace_size([fake_matrix(8, 4096)], hp_nt, 0) > thin


@pytest.mark.parametrize("mutate,code", [
    (lambda m, h: setattr(m, "rows", 0), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(m, "cols", -3), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(m, "grad", None), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(m, "weight_dtype", 7), dm.DM_ERR_UNSUPPORTED),
    (lambda m, h: setattr(h, "ns_steps", 0), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(h, "precision", 5), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(h, "scale_mode", 9), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(h, "scale_mode", 4), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(h, "lr", float("nan")), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(m, "row_energy", None), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: setattr(h, "ns_steps", dm.DM_MAX_NS_STEPS + 1), dm.DM_ERR_INVALID_ARG),
    (lambda m, h: dm.set_ns_coeffs(h, [(3.0, -4.0, 2.0), (1.0, float("inf"), 0.0)]),
     dm.DM_ERR_INVALID_ARG),
    (lambda m, h: dm.set_ns_coeffs(h, [(3.0, float("nan"), 2.0)]), dm.DM_ERR_INVALID_ARG),
])
def test_argument_errors_are_synchronous(mutate, code):
    m = fake_matrix(64, 96)
    hp = dm.dm_default_hparams()
    mutate(m, hp)
    # validated before any device call: these return without touching a GPU
    assert dm.dm_dimuon_step([m], hp, (0x100000, 1 << 30), stream=0) == code


@pytest.mark.parametrize("mode", [dm.DM_SCALE_NONE, dm.DM_SCALE_MOONSHOT, dm.DM_SCALE_JORDAN,
                                  dm.DM_SCALE_BERNSTEIN])
def test_every_scale_mode_is_accepted(mode):
    """Argument validation passes (the call then stops at the missing
    workspace, before any device work)."""
    m = fake_matrix(64, 96)
    hp = dm.dm_default_hparams(scale_mode=mode)
    assert dm.dm_muon_step([m], hp, (0, 0), stream=0) == dm.DM_ERR_WORKSPACE
    assert dm.dm_workspace_size([m], hp, 0) > 0


def test_launch_counts():
    """Kernel launches per step, from the planner (host-only)."""
    hp = dm.dm_default_hparams()
    big = [fake_matrix(4096, 4096)] * 8 + [fake_matrix(4096, 14336)] * 8
    # K1, K1b, 5 x 3 products
    assert dm.dm_step_launches(big, hp, 0) == 2 + 15
    # + K0, and K3a + K3
    assert dm.dm_step_launches(big, hp, 1) == 1 + 2 + 15 + 2
    # 448 rank-8 LoRA factors: the two-pass staged kernels (set-up, Gram,
    # iteration, apply), or one launch of the cluster kernel
    lora = [fake_matrix(8, 4096), fake_matrix(4096, 8)] * 224
    for m in lora:
        m.momentum_dtype = dm.DM_FP32
    assert dm.dm_step_launches(lora, hp, 1) == 4
    cl = dm.dm_default_hparams(debug_flags=dm.DM_DBG_THIN_CLUSTER)
    assert dm.dm_step_launches(lora, cl, 1) == 1
    # rank 2: the cluster kernel by default
    lora2 = [fake_matrix(2, 4096), fake_matrix(4096, 2)] * 224
    for m in lora2:
        m.momentum_dtype = dm.DM_FP32
    assert dm.dm_step_launches(lora2, hp, 1) == 1
    staged = dm.dm_default_hparams(debug_flags=dm.DM_DBG_THIN_STAGED)
    assert dm.dm_step_launches(lora2, staged, 1) == 4
    # rank 32 has no cluster kernel
    lora32 = [fake_matrix(32, 4096), fake_matrix(4096, 32)] * 224
    for m in lora32:
        m.momentum_dtype = dm.DM_FP32
    assert dm.dm_step_launches(lora32, hp, 1) == 4
    assert dm.dm_step_launches([], hp, 0) == 0


def test_coefficient_schedule_is_accepted():
    """A finite per-iteration schedule passes validation (the call then stops
    at the missing workspace); its length sets ns_steps; the default has none."""
    m = fake_matrix(64, 96)
    assert not dm.dm_default_hparams().ns_coeffs
    hp = dm.dm_default_hparams(ns_coeffs=[(3.4445, -4.775, 2.0315)] * 3 + [(1.875, -1.25, 0.375)])
    assert hp.ns_steps == 4 and abs(hp.ns_coeffs[9] - 1.875) < 1e-7
    assert dm.dm_muon_step([m], hp, (0, 0), stream=0) == dm.DM_ERR_WORKSPACE
    assert dm.dm_workspace_size([m], hp, 0) == dm.dm_workspace_size([m], dm.dm_default_hparams(), 0)


def test_workspace_errors():
    m = fake_matrix(64, 96)
    hp = dm.dm_default_hparams()
    need = dm.dm_workspace_size([m], hp, 0)
    assert dm.dm_muon_step([m], hp, (0, need), stream=0) == dm.DM_ERR_WORKSPACE
    assert dm.dm_muon_step([m], hp, (0x100010, need), stream=0) == dm.DM_ERR_WORKSPACE   # misaligned
    assert dm.dm_muon_step([m], hp, (0x100000, need - 1), stream=0) == dm.DM_ERR_WORKSPACE


def test_muon_ignores_missing_energies():
    m = fake_matrix(64, 96, energies=False)
    hp = dm.dm_default_hparams()
    assert dm.dm_workspace_size([m], hp, 0) > 0
    with pytest.raises(dm.DimuonError):
        dm.dm_workspace_size([m], hp, 1)


def test_header_constants_match_binding():
    """Every integer #define and enumerator of the header has the same value in
    the binding (a flag added on one side only would silently do nothing)."""
    text = open(HEADER).read()
    consts = {}
    for name, val in re.findall(r"^#define (DM_\w+) (0x[0-9a-fA-F]+|\d+)u?\b", text, flags=re.M):
        consts[name] = int(val, 0)
    for name, val in re.findall(r"\b(DM_[A-Z0-9_]+) = (\d+)", text):
        consts[name] = int(val)
    assert "DM_DBG_THIN_STAGED" in consts and "DM_ERR_NONFINITE" in consts
    for name, val in consts.items():
        assert hasattr(dm, name), f"binding lacks {name}"
        assert getattr(dm, name) == val, (name, getattr(dm, name), val)
    # debug flags are distinct bits
    bits = [v for k, v in consts.items() if k.startswith("DM_DBG_")]
    assert all(b & (b - 1) == 0 for b in bits) and len(set(bits)) == len(bits)


def test_checked_mode_sizes():
    """The checked-workspace mode adds a 256-byte canary after the header and
    after every region, and two launches (fill, check)."""
    hp = dm.dm_default_hparams()
    hpc = dm.dm_default_hparams(debug_flags=dm.DM_DBG_CANARY)
    mats = [fake_matrix(300, 500), fake_matrix(8, 4096)]
    assert dm.dm_workspace_size(mats, hpc, 1) >= dm.dm_workspace_size(mats, hp, 1) + 256 * 10
    assert dm.dm_step_launches(mats, hpc, 1) == dm.dm_step_launches(mats, hp, 1) + 2
    assert dm.dm_status_string(dm.DM_ERR_CANARY) == "workspace canary overwritten"
