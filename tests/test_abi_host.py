"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the headers declare, and rejects invalid arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_121_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in ("kda.h", "kda_testing.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"KDA_API[^;(]*?\b(kda_\w+)\s*\(", src))
    return names


def test_library_builds_and_loads():
    from gated_delta_rule_121_b200 import build
    build.build()
    L = kda.lib()
    assert L.kda_version() == 100


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"kda_fwd", "kda_decode_step", "kda_fwd_workspace_size", "kda_status_string",
            "kda_workspace_status", "kda_version"} <= names
    L = kda.lib()
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared but not exported"


def test_status_strings():
    for code in range(7):
        s = kda.kda_status_string(code)
        assert s.startswith("KDA_")
    assert "UNKNOWN" in kda.kda_status_string(99)


P = ctypes.c_void_p


def _fwd(**kw):
    a = dict(q=P(256), k=P(512), v=P(768), g=P(1024), beta=P(1280), init=None, out=P(1536), fin=None,
             B=1, T=64, H=2, dk=128, dv=128, cu=None, stream=None, dt=kda.KDA_BF16, ws=P(4096), wsb=256)
    a.update(kw)
    return kda.lib().kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["init"], a["out"], a["fin"], a["B"],
                             a["T"], a["H"], a["dk"], a["dv"], a["cu"], a["stream"], a["dt"], a["ws"], a["wsb"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=P(1282)), kda.KDA_ERR_INVALID_ARG),          # misaligned
    (dict(init=P(8)), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(B=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-5), kda.KDA_ERR_INVALID_ARG),
    (dict(dt=7), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(ws=None), kda.KDA_ERR_WORKSPACE),
    (dict(wsb=8), kda.KDA_ERR_WORKSPACE),
    (dict(cu=P(20)), kda.KDA_ERR_INVALID_ARG),
])
def test_fwd_rejects_invalid_arguments(kw, code):
    assert _fwd(**kw) == code


def test_fwd_rejects_more_than_2_31_tokens():
    """The batched token count B*T must fit the kernels' 32-bit token index."""
    assert _fwd(B=3, T=1 << 30, ws=P(4096), wsb=1024) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(B=1, T=(1 << 31), wsb=1024) == kda.KDA_ERR_UNSUPPORTED


def test_decode_rejects_invalid_arguments():
    L = kda.lib()
    ok = [P(256), P(512), P(768), P(1024), P(1280), P(1536), P(2048)]
    def call(ptrs, B=1, H=1, dk=128, dv=128, dt=kda.KDA_BF16):
        return L.kda_decode_step(*ptrs, B, H, dk, dv, None, dt)
    for i in range(7):
        bad = list(ok)
        bad[i] = None
        assert call(bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(ok)
    bad[5] = P(1540)
    assert call(bad) == kda.KDA_ERR_INVALID_ARG
    assert call(ok, dk=48) == kda.KDA_ERR_UNSUPPORTED
    assert call(ok, H=0) == kda.KDA_ERR_INVALID_ARG
    assert call(ok, B=0) == kda.KDA_OK          # no-op, no device work


def test_workspace_size_and_path_selection():
    assert kda.kda_fwd_workspace_size(2, 4096, 16, 128, 128) >= 16
    L = kda.lib()
    assert L.kda_testing_fwd_path(128, 128, kda.KDA_BF16) == 1
    assert L.kda_testing_fwd_path(128, 128, kda.KDA_F32) == 0
    assert L.kda_testing_fwd_path(16, 16, kda.KDA_BF16) == 0
    assert L.kda_testing_debug_floats() > 60000


def test_no_cpu_fallback_in_product_path():
    """The binding never imports the oracle and has no CPU code path."""
    src = open(os.path.join(ROOT, "gated_delta_rule_121_b200", "__init__.py")).read()
    assert "oracle" not in src
    assert "numpy" not in src


def test_new_entry_points_reject_invalid_arguments_on_the_host():
    L = kda.lib()
    fwd = [P(256), P(512), P(768), P(1024), P(1280), None, P(1536), P(2048), 1, 64, 2, 128, 128, None, None,
           kda.KDA_BF16]
    # checkpoints: interval must be a positive multiple of 64; a batched call needs B*floor(T/interval) slots
    assert L.kda_fwd_checkpoints(*fwd, P(4096), 100, 8, P(8192), 1 << 20) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_fwd_checkpoints(*fwd, P(4096), 0, 8, P(8192), 1 << 20) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_fwd_checkpoints(*fwd, P(4096), 64, 0, P(8192), 1 << 20) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_fwd_checkpoints(*fwd, P(4100), 64, 8, P(8192), 1 << 20) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_fwd_checkpoints(*fwd, P(4096), 64, 8, None, 0) == kda.KDA_ERR_WORKSPACE
    # segment pieces need square states
    seg = [P(256), P(512), P(768), P(1024), P(1280), P(1536), P(2048), P(2560), P(3072)]
    assert L.kda_segment_fwd(*seg, 1, 64, 2, 128, 64, None, None, kda.KDA_BF16, P(8192), 1024) == \
        kda.KDA_ERR_UNSUPPORTED
    assert L.kda_segment_fwd(*seg[:5], None, *seg[6:], 1, 64, 2, 128, 128, None, None, kda.KDA_BF16, P(8192),
                             1024) == kda.KDA_ERR_INVALID_ARG
    # composition and correction
    assert L.kda_state_compose(P(256), P(512), None, None, None, 2, 1, 1, 96, 128, 0, None) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_state_compose(None, None, None, None, None, 2, 1, 1, 128, 128, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_state_compose(None, None, None, None, None, 2, 0, 1, 128, 128, 0, None) == kda.KDA_OK
    assert L.kda_output_correct(P(256), P(512), P(768), P(1032), 1, 64, 2, 128, 128, None, None,
                                kda.KDA_BF16) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_output_correct(P(256), P(512), P(768), P(1024), 1, 0, 2, 128, 128, None, None,
                                kda.KDA_BF16) == kda.KDA_OK
    # context parallelism: n_seg >= 1, square states, a large enough workspace
    cp = fwd + [2]
    assert L.kda_fwd_cp(*fwd, 0, P(8192), 1 << 30) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_fwd_cp(*cp, P(8192), 64) == kda.KDA_ERR_WORKSPACE
    need = L.kda_fwd_cp_workspace_size(1, 64, 2, 128, 128, kda.KDA_BF16, 2)
    assert need >= 2 * 2 * 4 * 128 * 128 * 4  # four states per (segment, head)
    assert L.kda_cp_segments(2, 4096, 16, 148) == 3  # 32 chains: 3 x 32 blocks per pass
    assert L.kda_cp_segments(1, 65536, 96, 148) == 1


def test_kcp_module_has_no_oracle_or_cpu_path():
    src = open(os.path.join(ROOT, "gated_delta_rule_121_b200", "kcp.py")).read()
    assert "oracle" not in src.replace("oracle_ops", "") and "numpy" not in src
