"""C ABI checks that need no GPU: the library builds and loads, exports every function that
include/moba.h declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moba.h")

FAKE = ctypes.c_void_p(0x100000)  # 16-byte aligned, never dereferenced on these paths


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_moba_b200 import build, moba
    build.build()
    return moba.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moba_[a-z0-9_]+)\s*\(", text)))


def _cu(vals):
    return (ctypes.c_int32 * len(vals))(*vals)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "moba_attn_fwd" in names and "moba_centroids" in names and "moba_gate_topk" in names
    for n in names:
        assert hasattr(lib, n), n


def test_binding_lists_the_header(lib):
    from block_sparse_long_moba_b200 import moba
    assert sorted(moba.EXPORTS) == declared_functions()


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.moba_status_string(code).startswith(b"MOBA_")
    assert lib.moba_status_string(12345) == b"MOBA_UNKNOWN_STATUS"
    assert lib.moba_version() > 0


def test_workspace_bytes_valid_and_invalid(lib):
    ok = lib.moba_workspace_bytes(1, _cu([0, 131072]), 32, 8, 128, 4096, 12)
    assert ok > 0
    assert lib.moba_workspace_bytes(1, _cu([0, 1024]), 3, 2, 64, 128, 3) == 0      # Hq % Hkv
    assert lib.moba_workspace_bytes(1, _cu([0, 1024]), 2, 2, 96, 128, 3) == 0      # d
    assert lib.moba_workspace_bytes(1, _cu([0, 1024]), 2, 2, 64, 100, 3) == 0      # block
    assert lib.moba_workspace_bytes(1, _cu([0, 1024]), 2, 2, 64, 128, 0) == 0      # topk
    assert lib.moba_workspace_bytes(1, _cu([0, 1024]), 2, 2, 64, 128, 65) == 0     # topk max
    assert lib.moba_workspace_bytes(2, _cu([0, 10, 5]), 2, 2, 64, 128, 3) == 0     # decreasing
    assert lib.moba_workspace_bytes(1, _cu([1, 10]), 2, 2, 64, 128, 3) == 0        # cu[0] != 0
    # more varlen sequences or a larger problem need more workspace
    small = lib.moba_workspace_bytes(1, _cu([0, 4096]), 4, 4, 64, 128, 8)
    big = lib.moba_workspace_bytes(1, _cu([0, 8192]), 4, 4, 64, 128, 8)
    assert big > small > 0


def _attn(lib, cu, nseq, Hq=2, Hkv=2, d=64, B=128, topk=3, scale=0.125, ptr=FAKE,
          ws=FAKE, ws_bytes=1 << 40, lse=FAKE):
    return lib.moba_attn_fwd(ptr, ptr, ptr, ptr, cu, nseq, Hq, Hkv, d, B, topk,
                             ctypes.c_float(scale), None, None, ptr, lse, ws,
                             ctypes.c_size_t(ws_bytes), None)


def test_attn_fwd_host_side_errors(lib):
    cu = _cu([0, 1024])
    assert _attn(lib, _cu([0, 10, 5]), 2) == -1                 # cu_seqlens decreasing
    assert _attn(lib, cu, 1, d=96) == -2                        # unsupported head dim
    assert _attn(lib, cu, 1, Hq=3, Hkv=2) == -1                 # GQA groups must divide
    assert _attn(lib, cu, 1, scale=0.0) == -1                   # scale must be positive
    assert _attn(lib, cu, 1, ptr=None) == -1                    # null pointers
    assert _attn(lib, cu, 1, ptr=ctypes.c_void_p(0x100004)) == -1   # misaligned
    assert _attn(lib, cu, 1, ws=ctypes.c_void_p(0x100010)) == -1    # workspace not 256-aligned
    assert _attn(lib, cu, 1, ws_bytes=16) == -3                 # workspace too small
    assert _attn(lib, _cu([0, 0]), 1) == 0                      # empty input: nothing to do


def test_centroids_and_gate_host_side_errors(lib):
    cu = _cu([0, 1024])
    assert lib.moba_centroids(FAKE, FAKE, cu, 1, 2, 96, 128, FAKE, None) == -2
    assert lib.moba_centroids(FAKE, FAKE, cu, 1, 2, 64, 100, FAKE, None) == -2
    assert lib.moba_centroids(None, FAKE, cu, 1, 2, 64, 128, FAKE, None) == -1
    assert lib.moba_gate_topk(FAKE, FAKE, FAKE, cu, 1, 2, 2, 64, 128, 0, FAKE, None) == -1
    assert lib.moba_gate_topk(FAKE, None, FAKE, cu, 1, 2, 2, 64, 128, 3, FAKE, None) == -1
    assert lib.moba_gate_topk(FAKE, FAKE, FAKE, _cu([0, 0]), 1, 2, 2, 64, 128, 3, FAKE, None) == 0


def test_kconv_host_side_errors(lib):
    cu = _cu([0, 1024])
    kc = lib.moba_centroids_kconv
    assert kc(FAKE, None, 3, FAKE, cu, 1, 2, 64, 128, FAKE, None) == -1        # no weights
    assert kc(FAKE, FAKE, 0, FAKE, cu, 1, 2, 64, 128, FAKE, None) == -1        # width 0
    assert kc(FAKE, FAKE, 17, FAKE, cu, 1, 2, 64, 128, FAKE, None) == -2       # width > 16
    assert kc(FAKE, ctypes.c_void_p(0x100004), 3, FAKE, cu, 1, 2, 64, 128, FAKE, None) == -1
    assert kc(FAKE, FAKE, 3, FAKE, _cu([0, 0]), 1, 2, 64, 128, FAKE, None) == 0  # empty input
    af = lib.moba_attn_fwd_kconv
    assert af(FAKE, FAKE, FAKE, None, 3, FAKE, cu, 1, 2, 2, 64, 128, 3, ctypes.c_float(0.1),
              None, FAKE, FAKE, FAKE, ctypes.c_size_t(1 << 40), None) == -1
    assert af(FAKE, FAKE, FAKE, FAKE, 17, FAKE, cu, 1, 2, 2, 64, 128, 3, ctypes.c_float(0.1),
              None, FAKE, FAKE, FAKE, ctypes.c_size_t(1 << 40), None) == -2


def test_timing_classes_match_the_binding(lib):
    """moba_timing_read reports one entry per kernel class, in the binding's order (no GPU: with
    timing off nothing is recorded and no event is touched)."""
    from block_sparse_long_moba_b200 import moba
    assert lib.moba_timing_reset() == 0
    n = lib.moba_timing_read(None, None, 0)
    assert n == len(moba.KERNEL_CLASSES) == 13
    assert moba.KERNEL_CLASSES[-5:] == ["densify", "decode", "bwd_dkdv", "bwd_dq", "bwd_aux"]


@pytest.mark.parametrize("value,was_on", [("1", "1"), ("0", "0"), (None, "0")])
def test_timing_can_start_from_the_environment(value, was_on):
    """MOBA_TIMING=1 turns the timing hooks on when the library loads: in a fresh process,
    moba_timing_enable(0) then reports that timing was on (no GPU is touched)."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from block_sparse_long_moba_b200 import moba\n"
            "lib = moba.load_library()\n"
            "print(lib.moba_timing_enable(0), lib.moba_timing_enable(0))\n") % ROOT
    env = dict(os.environ)
    env.pop("MOBA_TIMING", None)
    if value is not None:
        env["MOBA_TIMING"] = value
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.split() == [was_on, "0"]
