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
    assert re.search(r"for \(.*<\s*\(1u? << 17\)", body) or "1 << 17" in body or "131072" in body
    assert "err" in body


def test_no_deliberate_traps():
    for name, text in _sources().items():
        assert "__trap" not in text, name
        assert not re.search(r'asm[^;]*"\s*trap', text), name
        assert "assert(" not in text, name
