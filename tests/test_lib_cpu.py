"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point declared in include/linattn.h, and answers host-only
queries (status strings, kernel choice, argument validation before launch)."""
import ctypes
import os
import re

import pytest
import torch

import recurrent_decode_la_b200 as la
from recurrent_decode_la_b200 import build as labuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "linattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(la_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    labuild.build()
    return la.load_library()


def test_every_declared_symbol_is_exported(lib):
    syms = _declared_symbols()
    assert "la_prefill" in syms and "la_decode_step" in syms and "la_state_init" in syms
    for name in syms:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(5):
        assert la.la_status_string(code)
    assert la.la_status_string(la.LA_ERR_TIMEOUT) == "device wait timed out"


def test_kernel_choice():
    assert la.la_prefill_path(torch.bfloat16, 128, 128, 64) == "tc"
    assert la.la_prefill_path(torch.bfloat16, 64, 64, 128) == "tc"
    assert la.la_prefill_path(torch.bfloat16, 128, 128, 128) == "tc"
    assert la.la_prefill_path(torch.bfloat16, 128, 128, 32) == "tc"
    assert la.la_prefill_path(torch.bfloat16, 64, 64, 16) == "tc"
    assert la.la_prefill_path(torch.bfloat16, 128, 128, 48) == "simt"
    assert la.la_prefill_path(torch.bfloat16, 96, 96, 64) == "simt"
    # with the token count: at most 16 tokens per unit run the few-token kernel
    assert la.la_prefill_kernel(torch.bfloat16, 16, 128, 128) == "short"
    assert la.la_prefill_kernel(torch.float32, 1, 5, 8) == "short"
    assert la.la_prefill_kernel(torch.bfloat16, 17, 128, 128) == "tc"
    assert la.la_prefill_kernel(torch.float32, 17, 128, 128) == "simt"
    assert la.la_prefill_kernel(torch.bfloat16, 8, 128, 6) == "simt"     # d_v not a multiple of 4
    assert la.la_prefill_kernel(torch.bfloat16, 8, 128, 80) == "simt"    # 20 float4 columns do not split 256 threads
    assert la.la_prefill_kernel(torch.bfloat16, 0, 128, 128) == "tc"     # packed, max_seqlen unknown
    assert la.la_prefill_path(torch.float32, 128, 128, 64) == "simt"
    assert la.la_prefill_path(torch.float32, 2, 2, 4) == "simt"
    assert la.la_prefill_path(torch.bfloat16, 256, 256, 64) == "unsupported"
    assert la.la_prefill_path(torch.float32, 128, 128, 256) == "unsupported"   # tiles exceed smem
    assert la.la_resolve_chunk(torch.bfloat16, 128, 128, 0) == 128
    assert la.la_resolve_chunk(torch.bfloat16, 128, 128, 96) == 96


def test_argument_checks_before_any_launch(lib):
    # all of these are rejected on the host: no device is touched
    assert lib.la_prefill(None, None, None, None, None, 1, 1, 1, 8, 64, 64, None, 0, 0, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG
    assert lib.la_prefill(None, None, None, None, None, 9, 1, 1, 8, 64, 64, None, 0, 0, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG
    assert lib.la_prefill(None, None, None, None, None, 1, -1, 1, 8, 64, 64, None, 0, 0, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG
    assert lib.la_prefill(None, None, None, None, None, 1, 2, 1, 8, 64, 64, 16, 1, 8, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG  # cu_seqlens needs B == 1
    assert lib.la_decode_step(None, None, None, None, None, 1, 1, 1, 64, 64, None) == la.LA_ERR_INVALID_ARG
    assert lib.la_decode_step(None, None, None, None, None, 1, 1, 1, 256, 64, None) == la.LA_ERR_UNSUPPORTED
    assert lib.la_state_init(None, None, 4, 8, 8, None) == la.LA_ERR_INVALID_ARG
    # empty work is a successful no-op, even with NULL pointers
    assert lib.la_prefill(None, None, None, None, None, 1, 0, 4, 8, 64, 64, None, 0, 0, 64, None, 0, None) == la.LA_OK
    assert lib.la_prefill(None, None, None, None, None, 1, 1, 4, 0, 64, 64, None, 0, 0, 64, None, 0, None) == la.LA_OK
    assert lib.la_state_init(None, None, 0, 8, 8, None) == la.LA_OK
    # the intra-sequence split needs workspace only for few, long, dense units
    assert lib.la_prefill_workspace_size(1, 8, 16, 8192, 128, 128, 0, 128) == 0
    assert lib.la_prefill_workspace_size(1, 1, 32, 131072, 128, 128, 0, 128) > 0
    # packed: never split; a work counter, then one int32 per sequence for the
    # longest-first order (2 to 4096 sequences)
    assert lib.la_prefill_workspace_size(1, 1, 32, 131072, 128, 128, 64, 128) == 512
    assert lib.la_prefill_workspace_size(1, 1, 32, 131072, 128, 128, 100, 128) == 768
    assert lib.la_prefill_workspace_size(1, 1, 32, 131072, 128, 128, 1, 128) == 256
    assert lib.la_prefill_workspace_size(1, 1, 32, 131072, 128, 128, 5000, 128) == 256
    assert lib.la_prefill_workspace_size(0, 1, 32, 131072, 128, 128, 0, 128) == 0    # fp32: CUDA-core path
    lib.la_selftest_wait_timeout.argtypes = [ctypes.c_double, ctypes.c_void_p]
    assert lib.la_selftest_wait_timeout(0.0, None) == la.LA_ERR_INVALID_ARG
    assert lib.la_selftest_wait_timeout(2e4, None) == la.LA_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors():
    x = torch.zeros(1, 1, 4, 8)
    with pytest.raises(ValueError):
        la.la_prefill(x, x, x, x.clone(), torch.zeros(1, 8, 8))


def test_missing_library_fails_loudly(tmp_path):
    """No CPU fallback: with the shared library absent, the first call raises."""
    code = (
        "import os, sys\n"
        f"os.environ['LINATTN_LIB'] = {str(tmp_path / 'absent.so')!r}\n"
        "import recurrent_decode_la_b200 as la\n"
        "try:\n"
        "    la.la_status_string(0)\n"
        "except OSError as e:\n"
        "    print('raised', e)\n"
        "    sys.exit(0)\n"
        "sys.exit(1)\n"
    )
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert r.returncode == 0, r.stdout + r.stderr
    assert "absent.so" in r.stdout


@pytest.mark.parametrize("case", ["small_state", "dense_state_for_packed", "short_cu", "packed_b2", "decode_state"])
def test_binding_checks_state_size_before_any_launch(case):
    """The kernels read and write units * d_k * d_v floats of state; the
    binding refuses a state of another size (and malformed packed offsets)
    with ValueError, before it touches the library or the device."""
    d = 8
    x = torch.zeros(2, 3, 5, d)
    with pytest.raises(ValueError):
        if case == "small_state":
            la.la_prefill(x, x, x, x.clone(), torch.zeros(2 * 3 - 1, d, d))
        elif case == "dense_state_for_packed":
            xp = torch.zeros(1, 3, 10, d)
            cu = torch.tensor([0, 4, 7, 10], dtype=torch.int32)           # 3 sequences x 3 heads
            la.la_prefill(xp, xp, xp, xp.clone(), torch.zeros(1 * 3, d, d), cu_seqlens=cu)
        elif case == "short_cu":
            xp = torch.zeros(1, 3, 10, d)
            la.la_prefill(xp, xp, xp, xp.clone(), torch.zeros(3, d, d), cu_seqlens=torch.tensor([0], dtype=torch.int32))
        elif case == "packed_b2":
            cu = torch.tensor([0, 5], dtype=torch.int32)
            la.la_prefill(x, x, x, x.clone(), torch.zeros(1 * 3, d, d), cu_seqlens=cu)
        else:
            t = torch.zeros(2, 3, d)
            la.la_decode_step(t, t, t, t.clone(), torch.zeros(2 * 3, d, d - 1))


def test_tuning_switches_are_read_once():
    """LINATTN_* switches are read on first use and never again: changing the
    environment later in the process changes nothing (a captured graph and a
    later direct call always agree)."""
    code = (
        "import os, sys\n"
        "os.environ['LINATTN_CHUNK'] = '64'\n"
        "import torch\n"
        "import recurrent_decode_la_b200 as la\n"
        "a = la.la_resolve_chunk(torch.bfloat16, 128, 128, 0)\n"
        "os.environ['LINATTN_CHUNK'] = '32'\n"
        "b = la.la_resolve_chunk(torch.bfloat16, 128, 128, 0)\n"
        "del os.environ['LINATTN_CHUNK']\n"
        "c = la.la_resolve_chunk(torch.bfloat16, 128, 128, 0)\n"
        "print(a, b, c)\n"
        "sys.exit(0 if (a, b, c) == (64, 64, 64) else 1)\n"
    )
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if not k.startswith("LINATTN_")}
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, env=env,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert r.returncode == 0, r.stdout + r.stderr
