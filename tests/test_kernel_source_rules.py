"""Source-level rules the kernels keep, checked on the CPU.

- Every pipeline wait is bounded: the mbarrier wait instruction appears in one helper
  (mbar_try_wait), and that helper is only called from the bounded loops next to it, which
  give up after a time limit, record TIMEOUT in the status header and return.
- The slot-pool claim of the calibration kernels is bounded the same way.
- No device code stops a kernel by trapping or by a failing device assert: failures are
  reported through the status header.
- No bulk or tensor copy uses cluster multicast.
"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_25_b200", "csrc")
SOURCES = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")))


def _text(path):
    with open(path) as f:
        return f.read()


def _strip_comments(src):
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def _function_body(src, name):
    """Text of the first function definition named `name` (brace-matched)."""
    m = re.search(r"\b" + re.escape(name) + r"\s*\([^;{]*\)\s*\{", src)
    assert m, name
    depth, i = 0, m.end() - 1
    while True:
        if src[i] == "{":
            depth += 1
        elif src[i] == "}":
            depth -= 1
            if depth == 0:
                return src[m.start():i + 1]
        i += 1


def test_sources_found():
    names = {os.path.basename(p) for p in SOURCES}
    assert {"bsa_common.cuh", "attn_fwd.cu", "block_mass.cu", "topp.cu"} <= names


def test_mbarrier_waits_only_through_the_bounded_helpers():
    common = _strip_comments(_text(os.path.join(CSRC, "bsa_common.cuh")))
    for path in SOURCES:
        src = _strip_comments(_text(path))
        waits = re.findall(r"mbarrier\.(?:try_wait|test_wait)", src)
        if os.path.basename(path) == "bsa_common.cuh":
            assert len(waits) == 1, path            # inside mbar_try_wait only
        else:
            assert not waits, path
            assert "mbar_try_wait(" not in src, path
    # mbar_try_wait's callers: the two bounded loops and nothing else
    callers = [m.start() for m in re.finditer(r"mbar_try_wait\(", common)]
    bodies = {n: _function_body(common, n) for n in ("mbar_wait_for", "mbar_wait_drain")}
    defn = _function_body(common, "mbar_try_wait")
    inside = 0
    for pos in callers:
        if common.find(defn) <= pos < common.find(defn) + len(defn):
            continue
        assert any(common.find(b) <= pos < common.find(b) + len(b) for b in bodies.values()), pos
        inside += 1
    assert inside >= 3
    for name, body in bodies.items():
        assert "globaltimer_ns()" in body and "limit" in body.lower(), name
        assert "record_status(" in body and "FLAG_TIMEOUT" in body, name
        assert "return false" in body, name


def test_every_kernel_wait_goes_through_the_limited_wrappers():
    """mbar_wait_for is called with an explicit limit only by the self-test wait (whose
    limit the caller gives, for the failure-detection test); every other wait uses
    mbar_wait (the library's 2 s limit) or mbar_wait_drain."""
    for path in SOURCES:
        if os.path.basename(path) == "bsa_common.cuh":
            continue
        src = _strip_comments(_text(path))
        if "mbar_wait_for(" in src:
            assert os.path.basename(path) == "selftest.cu", path
    common = _strip_comments(_text(os.path.join(CSRC, "bsa_common.cuh")))
    m = re.search(r"constexpr\s+uint64_t\s+kWaitLimitNs\s*=\s*(\d+)ull", common)
    assert m and int(m.group(1)) == 2_000_000_000


def test_slot_pool_claim_is_bounded():
    src = _strip_comments(_text(os.path.join(CSRC, "bsa_kernels.cuh")))
    body = _function_body(src, "claim_mass_slice")
    assert "globaltimer_ns()" in body and "kWaitLimitNs" in body
    assert "record_status(" in body and "return -1" in body


def test_no_trap_and_no_device_assert():
    for path in SOURCES:
        src = _strip_comments(_text(path))
        assert "__trap" not in src, path
        assert not re.search(r"\btrap\s*;", src), path
        assert not re.search(r"(?<![_\w])assert\s*\(", src), path   # static_assert is fine
        assert "__brkpt" not in src, path


def test_no_multicast_copies():
    for path in SOURCES:
        src = _strip_comments(_text(path))
        for stmt in re.findall(r"cp\.async\.bulk[^\"]*", src):
            assert "multicast" not in stmt, (path, stmt)
        assert ".multicast::cluster" not in src, path
