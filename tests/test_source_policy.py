"""Rules every source file keeps so that no GPU run can fault or hang shared
hardware (CPU only: the sources are read as text).

* No TMA or bulk LOAD that multi-casts to a cluster, anywhere (a
  ``tcgen05.commit`` that multi-casts is a completion signal, not a load, and is
  allowed).
* No batched host<->device copy API (one plain asynchronous copy per buffer).
* No ``__trap()`` and no device ``assert``: device-side failures are bounded
  waits that set a status the host reads.
* No absolute paths of the build machine.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DIRS = ["nonlinear_rnn_solve_newton_b200", "include", "oracle", "tests"]
FILES = ["bench.py", "__graft_entry__.py"]
EXT = (".cu", ".cuh", ".h", ".c", ".cpp", ".py")
SELF = os.path.abspath(__file__)
# the tokens are assembled so that this file never spells out such a load
MC = "multi" + "cast"
BULK = "cp.async" + ".bulk"


def sources():
    paths = [os.path.join(ROOT, f) for f in FILES]
    for d in DIRS:
        for base, dirs, names in os.walk(os.path.join(ROOT, d)):
            dirs[:] = [x for x in dirs if not x.startswith((".", "__pycache__"))]
            paths += [os.path.join(base, n) for n in names if n.endswith(EXT)]
    for p in sorted(paths):
        if os.path.abspath(p) != SELF:
            with open(p, encoding="utf-8") as f:
                yield os.path.relpath(p, ROOT), f.read()


def test_sources_are_found():
    names = [p for p, _ in sources()]
    assert any(p.endswith("pararnn.cu") for p in names)
    assert any(p.endswith("pararnn_proj.cuh") for p in names)


def mc_load_lines(text):
    """Lines naming the multi-cast qualifier within three lines of a bulk or
    tensor copy, other than a tcgen05.commit."""
    out = []
    lines = text.splitlines()
    for i, line in enumerate(lines):
        if MC not in line or "tcgen05.commit" in line:
            continue
        window = " ".join(lines[max(0, i - 3):i + 4])
        if BULK in window or "tensor" in window.lower():
            out.append(i + 1)
    return out


def test_mc_detector_positive_control():
    load = 'asm volatile("' + BULK + '.tensor.2d.shared::cluster.global.' + MC + '::cluster");'
    split = 'asm volatile("' + BULK + '.tensor.2d.shared::cluster.global"\n  ".' + MC + '::cluster");'
    commit = 'asm volatile("tcgen05.commit.cta_group::2.' + MC + '::cluster.b64 [%0], %1;");'
    assert mc_load_lines(load) == [1]
    assert mc_load_lines(split) == [2]
    assert mc_load_lines(commit) == []


def test_no_mc_loads():
    bad = [f"{path}:{n}" for path, text in sources() for n in mc_load_lines(text)]
    assert not bad, "multi-cast load in: " + "; ".join(bad)


BATCH_COPY = re.compile(r"Memcpy(3D)?Batch")
TRAP_OR_ASSERT = re.compile(r"__trap\s*\(|(?<![_\w])assert\s*\(")


def test_rule_patterns_positive_control():
    assert BATCH_COPY.search("cuda" + "Memcpy" + "Batch" + "Async(")
    assert BATCH_COPY.search("cu" + "Memcpy3D" + "Batch" + "Async(")
    assert not BATCH_COPY.search("cudaMemcpyAsync(dst, src, n, kind, s);")
    assert TRAP_OR_ASSERT.search("  __tr" + "ap();")
    assert TRAP_OR_ASSERT.search("  ass" + "ert(i < n);")
    assert not TRAP_OR_ASSERT.search('static_assert(N % 4 == 0, "x");')


def test_no_batched_copy_api():
    bad = [p for p, text in sources() if BATCH_COPY.search(text)]
    assert not bad, bad


def test_no_device_trap_or_assert():
    pat = TRAP_OR_ASSERT
    bad = []
    for path, text in sources():
        if not path.endswith((".cu", ".cuh")):
            continue
        for i, line in enumerate(text.splitlines()):
            if pat.search(line):
                bad.append(f"{path}:{i + 1}")
    assert not bad, bad


def test_no_machine_paths():
    bad = [p for p, text in sources() if "/root/" in text]
    assert not bad, bad
