"""Rules the CUDA sources keep (CPU, by reading them): every wait on an
mbarrier goes through the bounded helper, and no kernel traps on purpose."""

import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fourier_neural_spectral_fno_b200", "csrc")


def _sources():
    out = {}
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))):
        with open(path) as f:
            out[os.path.basename(path)] = f.read()
    return out


def test_mbarrier_waits_only_in_the_bounded_helper():
    srcs = _sources()
    assert "tc_util.cuh" in srcs
    for name, text in srcs.items():
        if name == "tc_util.cuh":
            continue
        assert "mbarrier.try_wait" not in text and "mbarrier.test_wait" not in text, name
        assert not re.search(r"\bmbar_try_wait(_sleep)?\s*\(", text), name
    helper = srcs["tc_util.cuh"]
    # the bounded wait: a fixed number of suspended attempts, then the error word
    body = helper[helper.index("bool mbar_wait("):]
    body = body[:body.index("\n}\n")]
    # a loop bounded by the library's wait limit (err[1], set by fno_set_wait_limit)
    # or, for the drains (err == NULL), by the default of 2^17 suspended polls
    assert re.search(r"for \(int i = 0; i < limit; \+\+i\)", body)
    assert "err ?" in body and "FNO_DEFAULT_WAIT_SPINS" in body
    assert re.search(r"#define FNO_DEFAULT_WAIT_SPINS \(1 << 17\)", helper)
    assert "err" in body
    api = srcs["fno_api.cu"]
    assert re.search(r"g_fno_device_error\[2\] = \{0, FNO_DEFAULT_WAIT_SPINS\}", api)


def test_no_deliberate_traps():
    for name, text in _sources().items():
        assert "__trap" not in text, name
        assert not re.search(r'asm[^;]*"\s*trap', text), name
        # device asserts (a failing one traps the kernel); static_assert is a
        # compile-time check and cannot reach the GPU
        assert not re.search(r"(?<!static_)\bassert\(", text), name
