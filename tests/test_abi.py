"""The C ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_87_b200 as gdr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "gated_delta.h")).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_library_loads_and_reports_abi_version():
    L = gdr.lib()
    assert L.kda_abi_version() == 1


def test_every_declared_symbol_is_exported():
    declared = _declared_symbols()
    assert len(declared) == len(gdr.EXPORTED_SYMBOLS)
    assert set(declared) == set(gdr.EXPORTED_SYMBOLS)
    L = ctypes.CDLL(gdr.library_path)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings():
    L = gdr.lib()
    for code in range(6):
        assert L.kda_status_string(code)
    assert L.kda_status_string(99) == b"unknown status"


def test_workspace_size_is_host_only_and_monotone():
    L = gdr.lib()
    a = L.kda_chunk_fwd_workspace_size(1, 4096, 32, 128, 128, 0, 1)
    b = L.kda_chunk_fwd_workspace_size(1, 8192, 32, 128, 128, 0, 1)
    assert 256 <= a <= b
    c = L.gdn_chunk_fwd_workspace_size(1, 4096, 16, 32, 128, 128, 0, 1)
    assert c == a


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _prefill(**over):
    L = gdr.lib()
    kw = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, o=FAKE + 4096, s0=None, sT=None,
              cu=None, num_seqs=0, B=1, T=64, H=2, d_k=128, d_v=128, io=1, ws=FAKE,
              ws_bytes=1 << 20)
    kw.update(over)
    return L.kda_chunk_fwd(kw["q"], kw["k"], kw["v"], kw["g"], kw["beta"], kw["o"], kw["s0"],
                           kw["sT"], kw["cu"], kw["num_seqs"], kw["B"], kw["T"], kw["H"],
                           kw["d_k"], kw["d_v"], kw["io"], kw["ws"], kw["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(q=None), gdr.KDA_ERR_INVALID_ARG),
    (dict(B=0), gdr.KDA_ERR_INVALID_ARG),
    (dict(d_k=96), gdr.KDA_ERR_UNSUPPORTED),
    (dict(d_v=32), gdr.KDA_ERR_UNSUPPORTED),
    (dict(io=7), gdr.KDA_ERR_INVALID_ARG),
    (dict(k=FAKE + 2), gdr.KDA_ERR_INVALID_ARG),
    (dict(o=FAKE), gdr.KDA_ERR_INVALID_ARG),
    (dict(ws=None), gdr.KDA_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), gdr.KDA_ERR_WORKSPACE),
    (dict(ws_bytes=16), gdr.KDA_ERR_WORKSPACE),
    (dict(cu=FAKE, num_seqs=2, B=2), gdr.KDA_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_arguments_on_host(over, status):
    assert _prefill(**over) == status
    assert gdr.lib().kda_last_error()


def test_gdn_rejects_indivisible_head_groups():
    L = gdr.lib()
    st = L.gdn_chunk_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4096, None, None, None, 0,
                         1, 64, 3, 4, 128, 128, 1, FAKE, 1 << 20, None)
    assert st == gdr.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((None,) + (FAKE,) * 6 + (4, 2, 128, 128, 1), gdr.KDA_ERR_INVALID_ARG),
    ((FAKE,) * 7 + (4, 2, 96, 128, 1), gdr.KDA_ERR_UNSUPPORTED),
    ((FAKE,) * 7 + (4, 2, 128, 128, 1), gdr.KDA_ERR_INVALID_ARG),  # o aliases the inputs
    ((FAKE,) * 5 + (FAKE + 8,) + (FAKE + 8,) + (4, 2, 128, 128, 1), gdr.KDA_ERR_INVALID_ARG),
    ((FAKE,) * 3 + (FAKE + 2,) + (FAKE,) + (FAKE + 4096,) + (FAKE + 8192,) + (4, 2, 128, 128, 1),
     gdr.KDA_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_on_host(args, status):
    L = gdr.lib()
    assert L.kda_decode_step(*args, None) == status


def test_binding_has_no_cpu_path():
    """The product binding never imports the oracle."""
    src = open(os.path.join(ROOT, "gated_delta_rule_87_b200", "__init__.py")).read()
    assert "oracle" not in re.sub(r'""".*?"""', "", src, flags=re.S)


def _prefill_ex(order=0, slots=None, num_slots=0, **over):
    L = gdr.lib()
    kw = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, o=FAKE + 4096, ws=FAKE, ws_bytes=1 << 20)
    kw.update(over)
    return L.kda_chunk_fwd_ex(kw["q"], kw["k"], kw["v"], kw["g"], kw["beta"], kw["o"], None, None,
                              slots, num_slots, None, 0, 1, 64, 2, 128, 128, order, 1, kw["ws"],
                              kw["ws_bytes"], None)


@pytest.mark.parametrize("kw", [
    dict(order=2), dict(order=-1),                  # no such decay order
    dict(slots=FAKE + 2, num_slots=4),              # misaligned slot array
    dict(slots=FAKE, num_slots=-1),                 # negative pool size
])
def test_prefill_ex_rejects_bad_arguments_on_host(kw):
    assert _prefill_ex(**kw) == gdr.KDA_ERR_INVALID_ARG
    assert gdr.lib().kda_last_error()


def _recurrent(order=0, slots=None, num_slots=0, N=4, T=3, ptr=FAKE, o=FAKE + 8192):
    L = gdr.lib()
    return L.kda_recurrent_fwd(ptr, FAKE, FAKE, FAKE, FAKE, o, FAKE + 16384, slots, num_slots,
                               N, T, 2, 128, 128, order, 1, None)


@pytest.mark.parametrize("kw,status", [
    (dict(order=5), gdr.KDA_ERR_INVALID_ARG),
    (dict(slots=FAKE + 1, num_slots=3), gdr.KDA_ERR_INVALID_ARG),
    (dict(slots=FAKE, num_slots=-3), gdr.KDA_ERR_INVALID_ARG),
    (dict(T=-1), gdr.KDA_ERR_INVALID_ARG),
    (dict(ptr=None), gdr.KDA_ERR_INVALID_ARG),
    (dict(o=FAKE), gdr.KDA_ERR_INVALID_ARG),        # o aliases q
])
def test_recurrent_rejects_bad_arguments_on_host(kw, status):
    assert _recurrent(**kw) == status


def test_recurrent_without_tokens_launches_nothing():
    """N = 0 or T = 0 returns before any CUDA call (works without a GPU)."""
    assert _recurrent(N=0, ptr=None) == gdr.KDA_OK
    assert _recurrent(T=0, ptr=None) == gdr.KDA_OK


def test_gdn_recurrent_rejects_indivisible_head_groups():
    L = gdr.lib()
    st = L.gdn_recurrent_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8192, FAKE + 16384, None, 0,
                             4, 2, 3, 4, 128, 128, 1, None)
    assert st == gdr.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((FAKE, None, 8, FAKE + 4096, 4, 2, 128, 128), gdr.KDA_ERR_INVALID_ARG),   # no slots
    ((FAKE, FAKE, 8, FAKE, 4, 2, 128, 128), gdr.KDA_ERR_INVALID_ARG),          # pool == out
    ((FAKE + 4, FAKE, 8, FAKE + 4096, 4, 2, 128, 128), gdr.KDA_ERR_INVALID_ARG),  # misaligned
    ((FAKE, FAKE, -1, FAKE + 4096, 4, 2, 128, 128), gdr.KDA_ERR_INVALID_ARG),  # negative pool
    ((FAKE, FAKE, 8, FAKE + 4096, 4, 2, 96, 128), gdr.KDA_ERR_UNSUPPORTED),
    ((None, None, 0, None, 0, 2, 128, 128), gdr.KDA_OK),                       # nothing to copy
])
def test_state_gather_validation(args, status):
    assert gdr.lib().kda_state_gather(*args, None) == status


def test_state_scatter_validation():
    L = gdr.lib()
    assert L.kda_state_scatter(FAKE, FAKE + 4096, None, 8, 4, 2, 128, 128, None) == \
        gdr.KDA_ERR_INVALID_ARG
    assert L.kda_state_scatter(None, None, None, 0, 0, 2, 128, 128, None) == gdr.KDA_OK


def test_selftest_wait_timeout_validates_on_host():
    """Argument checks run before the device is touched (no GPU needed)."""
    L = gdr.lib()
    assert L.kda_selftest_wait_timeout(None, 16, None) == gdr.KDA_ERR_INVALID_ARG
    dummy = ctypes.c_void_p(256)  # never dereferenced: the bound check fails first
    assert L.kda_selftest_wait_timeout(dummy, 0, None) == gdr.KDA_ERR_INVALID_ARG
    assert L.kda_selftest_wait_timeout(dummy, 5000, None) == gdr.KDA_ERR_INVALID_ARG


def test_checked_build_exports_the_same_symbols():
    """The bounds-checked build is the same library: same symbols, same ABI."""
    L = ctypes.CDLL(gdr.checked_library_path)
    for name in _declared_symbols():
        assert hasattr(L, name), name
    with gdr.use_library(gdr.checked_library_path) as C:
        assert C.kda_abi_version() == 1
        assert gdr.bounds_checked()
        assert C.kda_bounds_violations(None, None) == gdr.KDA_ERR_INVALID_ARG
    assert not gdr.bounds_checked()
    assert gdr.lib().kda_bounds_violations(None, None) == gdr.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("over,status", [
    (dict(T=0), gdr.KDA_ERR_INVALID_ARG),
    (dict(pieces=65), gdr.KDA_ERR_INVALID_ARG),
    (dict(q=None), gdr.KDA_ERR_INVALID_ARG),
    (dict(io=7), gdr.KDA_ERR_INVALID_ARG),
    (dict(d_k=96), gdr.KDA_ERR_UNSUPPORTED),
    (dict(buf=None), gdr.KDA_ERR_WORKSPACE),
    (dict(buf=FAKE + 16), gdr.KDA_ERR_WORKSPACE),
    (dict(buf_bytes=1024), gdr.KDA_ERR_WORKSPACE),
])
def test_streamed_prefill_rejects_bad_arguments_on_host(over, status):
    L = gdr.lib()
    kw = dict(q=FAKE, B=1, T=256, H=2, d_k=128, d_v=128, io=1, pieces=4, buf=FAKE,
              buf_bytes=1 << 30)
    kw.update(over)
    st = L.kda_chunk_fwd_host(kw["q"], FAKE, FAKE, FAKE, FAKE, FAKE, None, None, kw["B"], kw["T"],
                              kw["H"], kw["d_k"], kw["d_v"], kw["io"], kw["pieces"], kw["buf"],
                              kw["buf_bytes"], None)
    assert st == status
    assert L.kda_last_error()


def test_streamed_prefill_buffer_size():
    L = gdr.lib()
    a = L.kda_chunk_fwd_host_buffer_size(1, 4096, 32, 128, 128, 1, 8)
    b = L.kda_chunk_fwd_host_buffer_size(1, 8192, 32, 128, 128, 1, 8)
    # at least the staged inputs and output: q, k, v, o bf16 and g fp32 per token-head
    assert a >= 4096 * 32 * (4 * 128 * 2 + 128 * 4) and b > a
    assert L.kda_chunk_fwd_host_buffer_size(1, 4096, 32, 128, 128, 1, 65) == 0
    assert L.kda_chunk_fwd_host_buffer_size(1, 0, 32, 128, 128, 1, 8) == 0
