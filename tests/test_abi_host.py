"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/mla_decode.h declares, and rejects bad arguments before
touching a device."""

import ctypes
import os
import re

import pytest

from mla_paged_kv_05_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "mla_decode.h")) as f:
        text = f.read()
    return set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text))


def test_header_declares_the_binding_table():
    assert declared_symbols() == set(_lib.SIGNATURES)


def test_flag_bits_agree_between_header_binding_and_device_code():
    """The device-flag bits are spelled three times: the C header, the Python
    binding and the kernels' constants. They must be the same bits."""
    with open(os.path.join(ROOT, "include", "mla_decode.h")) as f:
        header = dict((k, int(v)) for k, v in re.findall(r"#define MLA_FLAG_(\w+)\s+(\d+)", f.read()))
    with open(os.path.join(ROOT, "mla_paged_kv_05_b200", "csrc", "mla_common.cuh")) as f:
        device = dict((k, int(v)) for k, v in re.findall(r"constexpr int kFlag(\w+) = (\d+);", f.read()))
    binding = {k[len("FLAG_"):]: v for k, v in vars(_lib).items() if k.startswith("FLAG_")}
    assert header == binding
    camel = {"TIMEOUT": "Timeout", "BAD_SEQLEN": "BadSeqlen", "BAD_PAGE": "BadPage", "BAD_PREFIX": "BadPrefix",
             "PLAN_MISMATCH": "PlanMismatch"}
    assert set(camel) == set(header)
    assert {camel[k]: v for k, v in header.items()} == device
    bits = list(header.values())
    assert all(b & (b - 1) == 0 for b in bits) and len(set(bits)) == len(bits)   # distinct single bits


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.mla_version().decode().startswith("mla_decode")


def _plan(lib, batch=1, max_pages=4, q_len=1, heads=16, kv=0, sm_budget=0):
    nbytes = ctypes.c_size_t(0)
    splits = ctypes.c_int(0)
    st = lib.mla_decode_plan(None, None, 0, batch, max_pages, q_len, heads, kv, sm_budget, None,
                             ctypes.byref(nbytes), ctypes.byref(splits), None)
    return st, lib.mla_get_last_error().decode()


@pytest.mark.parametrize("kw,status,msg", [
    (dict(batch=-1), _lib.MLA_ERR_INVALID_ARG, "batch"),
    (dict(max_pages=0), _lib.MLA_ERR_INVALID_ARG, "max_pages"),
    (dict(q_len=0), _lib.MLA_ERR_UNSUPPORTED, "q_len"),
    (dict(q_len=5), _lib.MLA_ERR_UNSUPPORTED, "q_len"),
    (dict(heads=0), _lib.MLA_ERR_UNSUPPORTED, "heads"),
    (dict(heads=129), _lib.MLA_ERR_UNSUPPORTED, "heads"),
    (dict(kv=7), _lib.MLA_ERR_INVALID_ARG, "kv_dtype"),
    (dict(sm_budget=-2), _lib.MLA_ERR_INVALID_ARG, "sm_budget"),
])
def test_plan_rejects_bad_shapes_on_the_host(lib, kw, status, msg):
    st, err = _plan(lib, **kw)
    assert st == status and msg in err, (st, err)


def _plan_bt(lib, block_table, num_pages, batch=1, max_pages=4):
    nbytes = ctypes.c_size_t(0)
    st = lib.mla_decode_plan(None, block_table, num_pages, batch, max_pages, 1, 16, 0, 0, None,
                             ctypes.byref(nbytes), None, None)
    return st, lib.mla_get_last_error().decode()


@pytest.mark.parametrize("bt,num_pages,msg", [
    (0x1002, 8, "block_table must be 4-byte aligned"),
    (0x1000, 0, "num_pages"),
    (0x1000, 2 ** 31, "num_pages"),
])
def test_plan_checks_the_block_table_arguments_on_the_host(lib, bt, num_pages, msg):
    # The block table is optional (NULL: no page-id check in the planner); when
    # it is given, its alignment and the pool size it indexes are checked
    # before anything touches a device.
    st, err = _plan_bt(lib, bt, num_pages)
    assert st == _lib.MLA_ERR_INVALID_ARG and msg in err, (st, err)


def test_plan_rejects_a_cost_line_beyond_int32(lib):
    st, err = _plan(lib, batch=1 << 16, max_pages=1 << 14)
    assert st == _lib.MLA_ERR_UNSUPPORTED and "2^30" in err, (st, err)


def test_plan_requires_workspace_bytes_pointer(lib):
    st = lib.mla_decode_plan(None, None, 0, 1, 4, 1, 16, 0, 0, None, None, None, None)
    assert st == _lib.MLA_ERR_INVALID_ARG
    assert "workspace_bytes" in lib.mla_get_last_error().decode()


def _run(lib, **kw):
    a = dict(q=None, kv=None, num_pages=1, kv_dtype=0, bt=None, sl=None, out=None, lse=None, batch=1,
             max_pages=4, q_len=1, heads=16, scale=0.07, ws=None, ws_bytes=0, phases=3)
    a.update(kw)
    st = lib.mla_decode_run_phases(a["q"], a["kv"], a["num_pages"], a["kv_dtype"], a["bt"], a["sl"], a["out"],
                                   a["lse"], a["batch"], a["max_pages"], a["q_len"], a["heads"], a["scale"],
                                   a["ws"], a["ws_bytes"], a["phases"], None)
    return st, lib.mla_get_last_error().decode()


@pytest.mark.parametrize("kw,status,msg", [
    (dict(phases=0), _lib.MLA_ERR_INVALID_ARG, "phases"),
    (dict(phases=8), _lib.MLA_ERR_INVALID_ARG, "phases"),
    (dict(scale=0.0), _lib.MLA_ERR_INVALID_ARG, "scale"),
    (dict(scale=float("nan")), _lib.MLA_ERR_INVALID_ARG, "scale"),
    (dict(num_pages=0), _lib.MLA_ERR_INVALID_ARG, "num_pages"),
    (dict(q_len=9), _lib.MLA_ERR_UNSUPPORTED, "q_len"),
])
def test_run_rejects_bad_arguments_on_the_host(lib, kw, status, msg):
    st, err = _run(lib, **kw)
    assert st == status and msg in err, (st, err)


def test_error_message_is_per_call(lib):
    _plan(lib, q_len=0)
    assert lib.mla_get_last_error().decode()
    lib.mla_set_wait_timeout_ns(1000)
    lib.mla_set_wait_timeout_ns(10 ** 9)


def test_read_device_flag_rejects_null(lib):
    flag = ctypes.c_int(0)
    assert lib.mla_read_device_flag(None, ctypes.byref(flag), None) == _lib.MLA_ERR_INVALID_ARG


def _append(lib, **kw):
    a = dict(src=0x1000, cache=0x2000, num_pages=8, kv_dtype=0, bt=0x3000, sl=0x4000, batch=1, max_pages=4,
             q_len=1, flag=None)
    a.update(kw)
    st = lib.mla_cache_append(a["src"], a["cache"], a["num_pages"], a["kv_dtype"], a["bt"], a["sl"], a["batch"],
                              a["max_pages"], a["q_len"], a["flag"], None)
    return st, lib.mla_get_last_error().decode()


@pytest.mark.parametrize("kw,status,msg", [
    (dict(q_len=0), _lib.MLA_ERR_UNSUPPORTED, "q_len"),
    (dict(q_len=5), _lib.MLA_ERR_UNSUPPORTED, "q_len"),
    (dict(kv_dtype=3), _lib.MLA_ERR_INVALID_ARG, "kv_dtype"),
    (dict(num_pages=0), _lib.MLA_ERR_INVALID_ARG, "num_pages"),
    (dict(src=None), _lib.MLA_ERR_INVALID_ARG, "kv_new is NULL"),
    (dict(src=0x1008), _lib.MLA_ERR_INVALID_ARG, "kv_new must be 16-byte aligned"),
    (dict(bt=0x3002), _lib.MLA_ERR_INVALID_ARG, "block_table must be 4-byte aligned"),
    (dict(flag=0x5001), _lib.MLA_ERR_INVALID_ARG, "flag must be 4-byte aligned"),
])
def test_append_rejects_bad_arguments_on_the_host(lib, kw, status, msg):
    st, err = _append(lib, **kw)
    assert st == status and msg in err, (st, err)


def test_append_of_an_empty_batch_is_a_no_op(lib):
    st, _ = _append(lib, batch=0, src=None, cache=None, bt=None, sl=None)
    assert st == _lib.MLA_OK


@pytest.mark.parametrize("fn", ["mla_absorb_q", "mla_project_out"])
@pytest.mark.parametrize("args,status,msg", [
    ((0x1000, 0x2000, 0x3000, -1, 4), _lib.MLA_ERR_UNSUPPORTED, "n_tokens"),
    ((0x1000, 0x2000, 0x3000, 4, 0), _lib.MLA_ERR_UNSUPPORTED, "heads"),
    ((0x1000, 0x2000, 0x3000, 4, 129), _lib.MLA_ERR_UNSUPPORTED, "heads"),
    ((None, 0x2000, 0x3000, 4, 4), _lib.MLA_ERR_INVALID_ARG, "is NULL"),
    ((0x1000, 0x2008, 0x3000, 4, 4), _lib.MLA_ERR_INVALID_ARG, "16-byte aligned"),
])
def test_projections_reject_bad_arguments_on_the_host(lib, fn, args, status, msg):
    st = getattr(lib, fn)(*args, None, None)
    err = lib.mla_get_last_error().decode()
    assert st == status and msg in err, (st, err)


@pytest.mark.parametrize("fn", ["mla_absorb_q", "mla_project_out"])
def test_projection_of_no_tokens_is_a_no_op(lib, fn):
    assert getattr(lib, fn)(None, None, None, 0, 8, None, None) == _lib.MLA_OK
