"""The C-ABI library loads on a CPU-only host, exports every symbol that
include/sba.h declares, validates arguments on the host, and its host-side
geometry agrees with the oracle. No device call is made here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sba():
    import block_sparse_attention_sba_b200 as m
    return m


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "sba.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sba_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for s in ["sba_reorder", "sba_build_mask", "sba_attention", "sba_unreorder",
              "sba_plan_create", "sba_check_device_status", "sba_status_string"]:
        assert s in syms


def test_library_exports_every_declared_symbol(sba):
    lib = ctypes.CDLL(sba.LIB_PATH)
    for s in _declared_symbols():
        assert hasattr(lib, s), f"{s} declared in sba.h but not exported"
    assert set(_declared_symbols()) == set(sba.EXPORTED)


def test_status_strings(sba):
    for code in range(-6, 1):
        assert sba.sba_status_string(code).startswith("SBA_")


GEOMS = [
    (1, 2, 4, 8, 8, 64, (4, 4, 4), "f32"),
    (1, 8, 8, 16, 16, 64, (4, 4, 4), "bf16"),
    (1, 40, 21, 30, 52, 128, (2, 8, 8), "bf16"),
    (1, 24, 33, 45, 80, 128, (2, 8, 8), "bf16"),
    (2, 3, 5, 9, 7, 64, (2, 4, 8), "bf16"),
]


@pytest.mark.parametrize("B,H,T,Hh,W,d,cube,dt", GEOMS)
def test_plan_geometry_matches_oracle(sba, B, H, T, Hh, W, d, cube, dt):
    plan = sba.Plan(B, H, T, Hh, W, d, cube, dt)
    g = oracle.Geom(T, Hh, W, *cube)
    inf = plan.info
    assert (inf.nT, inf.nH, inf.nW, inf.nb, inf.bs, inf.Npad) == (g.nT, g.nH, g.nW, g.nb, g.bs, g.Npad)
    assert inf.rows == B * H * g.nb and inf.words == (g.nb + 31) // 32
    assert inf.max_nnz == inf.rows * g.nb
    assert inf.workspace_bytes >= 256 + 2 * inf.rows * d * 4


@pytest.mark.parametrize("T,Hh,W,cube", [(4, 8, 8, (4, 4, 4)), (5, 9, 7, (2, 4, 8)),
                                         (21, 30, 52, (2, 8, 8)), (3, 3, 3, (1, 8, 8))])
def test_host_permutation_matches_oracle(sba, T, Hh, W, cube):
    plan = sba.Plan(1, 1, T, Hh, W, 64, cube, "bf16")
    got = np.array(sba.sba_perm_export(plan.handle, T * Hh * W))
    assert np.array_equal(got, oracle.slot_of_token(oracle.Geom(T, Hh, W, *cube)))


@pytest.mark.parametrize("T,Hh,W,cube", [(4, 8, 8, (4, 4, 4)), (5, 9, 7, (2, 4, 8)),
                                         (21, 30, 52, (2, 8, 8)), (3, 10, 6, (1, 8, 8))])
def test_host_hilbert_permutation_matches_oracle(sba, T, Hh, W, cube):
    plan = sba.Plan(1, 1, T, Hh, W, 64, cube, "bf16", order="hilbert")
    g = oracle.Geom(T, Hh, W, *cube, order="hilbert")
    assert (plan.info.nb, plan.info.Npad) == (g.nb, g.Npad)
    got = np.array(sba.sba_perm_export(plan.handle, T * Hh * W))
    assert np.array_equal(got, oracle.slot_of_token(g))


def test_hilbert_reorder_requires_the_workspace(sba):
    plan = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16", order="hilbert")
    fake = 1 << 20
    with pytest.raises(sba.SbaError) as e:
        sba.sba_reorder(plan.handle, fake, None, None, fake, None, None, None, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_unreorder(plan.handle, fake, fake, None, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), -2),                       # untuned head dim
    (dict(cube=(2, 4, 4)), -2),             # block of 32
    (dict(dt="f32", d=128), -2),
    (dict(T=0), -1),
    (dict(H=300), -4),
    (dict(B=40, H=256), -4),                # B*H above 8192
    (dict(T=200, Hh=64, W=64), -4),         # too many blocks per head
])
def test_plan_rejects_bad_geometry(sba, kw, code):
    args = dict(B=1, H=2, T=4, Hh=8, W=8, d=64, cube=(4, 4, 4), dt="bf16")
    args.update(kw)
    with pytest.raises(sba.SbaError) as e:
        sba.Plan(args["B"], args["H"], args["T"], args["Hh"], args["W"], args["d"], args["cube"],
                 args["dt"])
    assert e.value.status == code


def test_plan_rejects_unaligned_strides(sba):
    with pytest.raises(sba.SbaError) as e:
        sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16", strides=(4 * 8 * 8 * 64 * 2, 4 * 8 * 8 * 64, 68))
    assert e.value.status == sba.SBA_ERR_INVALID_ARG


def test_calls_validate_before_any_launch(sba):
    plan = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16")
    h = plan.handle
    fake = 1 << 20  # never dereferenced: validation fails first
    with pytest.raises(sba.SbaError) as e:
        sba.sba_reorder(h, fake, None, None, None, None, None, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_reorder(h, fake + 8, None, None, fake, None, None, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG     # misaligned
    for bad_p in ([0.0, 0.5], [0.5, 1.5], [float("nan"), 0.5]):
        with pytest.raises(sba.SbaError) as e:
            sba.sba_build_mask(h, fake, fake, bad_p, 1, fake, fake, fake, fake, fake, fake, stream=0)
        assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_build_mask(h, fake, fake, [0.5, 0.5], -1, fake, fake, fake, fake, fake, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_attention(h, fake, fake, fake, fake, fake, fake, fake, None, 7, None, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_attention(h, fake, fake, fake, fake, fake, None, fake, None, sba.SBA_SCHED_LPT,
                          None, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    with pytest.raises(sba.SbaError) as e:
        sba.sba_debug_timeout_probe(h, fake, 10, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    assert "must" in sba.sba_last_error()


def test_binding_has_no_fallback_path():
    """The package is the C ABI plus marshalling: it must not import the
    oracle or any compute library."""
    src = open(os.path.join(ROOT, "block_sparse_attention_sba_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("no fallback", "")
    assert "numpy" not in src and "scaled_dot_product" not in src


def test_stripe_mask_validates_before_any_launch(sba):
    plan = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16")
    h = plan.handle
    fake = 1 << 20  # never dereferenced: validation fails first
    ok = (3, -1, 0, 5, -2, 0)
    for bad in [(-1, 0, 0, 1, 0, 0), (1, 0, -2, 1, 0, 0), (1, 0, 0, -3, 0, 0), (1, 0, 0, 1, 0, -1),
                (1, 40000, 0, 1, 0, 0), (1, 0, 0, 1, -40000, 0)]:
        with pytest.raises(sba.SbaError) as e:
            sba.sba_build_stripe_mask(h, [ok, bad], fake, fake, fake, fake, fake, fake, stream=0)
        assert e.value.status == sba.SBA_ERR_INVALID_ARG, bad
    with pytest.raises(sba.SbaError) as e:
        sba.sba_build_stripe_mask(h, [ok, ok], fake, fake, fake, fake, fake, fake + 8, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG  # misaligned workspace
    hplan = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16", order="hilbert")
    with pytest.raises(sba.SbaError) as e:
        sba.sba_build_stripe_mask(hplan.handle, [ok, ok], fake, fake, fake, fake, fake, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_UNSUPPORTED
    assert "cube" in sba.sba_last_error()


def test_stripe_struct_matches_the_header(sba):
    import ctypes
    assert ctypes.sizeof(sba.sba_stripe) == 24
    text = open(os.path.join(ROOT, "include", "sba.h")).read()
    assert "int32_t Tw, To, Ts;" in text and "int32_t Sw, So, Ss;" in text
    assert [f[0] for f in sba.sba_stripe._fields_] == ["Tw", "To", "Ts", "Sw", "So", "Ss"]


def test_lowbit_calls_validate_before_any_launch(sba):
    fake = 1 << 20
    plan64 = sba.Plan(1, 2, 8, 16, 16, 64, (4, 4, 4), "bf16")
    with pytest.raises(sba.SbaError) as e:
        sba.sba_attention_lowbit(plan64.handle, fake, fake, fake, fake, fake, fake, fake, fake,
                                 fake, None, None, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_UNSUPPORTED
    plan = sba.Plan(1, 2, 5, 20, 19, 128, (2, 8, 8), "bf16")
    with pytest.raises(sba.SbaError) as e:
        sba.sba_attention_lowbit(plan.handle, fake, fake, fake, fake, fake, fake, fake, None,
                                 fake, None, None, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG  # work_order is required
    with pytest.raises(sba.SbaError) as e:
        sba.sba_attention_lowbit(plan.handle, fake, fake, fake + 8, fake, fake, fake, fake, fake,
                                 fake, None, None, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG  # misaligned codes
    planf = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "f32")
    with pytest.raises(sba.SbaError) as e:
        sba.sba_smooth_v(planf.handle, fake, fake, fake, fake, fake, stream=0)
    assert e.value.status == sba.SBA_ERR_UNSUPPORTED
