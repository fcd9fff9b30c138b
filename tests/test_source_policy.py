"""Source rules the CUDA code keeps, checked on the text of the sources (CPU).

- Every wait in device code is bounded: the PTX polls (mbarrier try_wait, the
  acquire load of a hand-off flag) occur only inside the three helpers of
  gdn_sm100.cuh, each a rolled loop over an iteration limit that the caller
  must pass (no default), and no source holds an unconditional loop.
- No device code stops a kernel by force: no trap instruction, no __trap(),
  no device assert.
"""
import pathlib
import re

import pytest

ROOT = pathlib.Path(__file__).resolve().parent.parent
CSRC = ROOT / "gated_deltanet_scan_chunked_b200" / "csrc"
SOURCES = sorted(p for p in CSRC.iterdir() if p.suffix in (".cu", ".cuh", ".h"))
HELPERS = CSRC / "gdn_sm100.cuh"
BOUNDED = ("mbar_wait", "mbar_wait_cluster", "wait_flag_ge")


def _strip_comments(text):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def _function_body(text, name):
    """Signature and body of the first definition of `name` in `text`."""
    m = re.search(r"\b(bool|void|unsigned long long|uint32_t)\s+%s\s*\(" % name, text)
    assert m, name
    i = text.index("{", m.end())
    depth = 0
    for j in range(i, len(text)):
        depth += {"{": 1, "}": -1}.get(text[j], 0)
        if depth == 0:
            return text[m.start():i], text[i:j + 1]
    raise AssertionError("unbalanced braces in " + name)


def test_sources_found():
    names = {p.name for p in SOURCES}
    assert {"gdn_sm100.cuh", "gdn_prefill_scan.cu", "gdn_decode.cu"} <= names


@pytest.mark.parametrize("name", BOUNDED)
def test_wait_helpers_are_bounded_rolled_loops(name):
    sig, body = _function_body(_strip_comments(HELPERS.read_text()), name)
    # the limit is a plain parameter: every call site has to give one
    assert re.search(r"uint32_t\s+max_iter\s*\)", sig), sig
    assert "=" not in sig, "no default limit: " + sig
    assert re.search(r"#pragma unroll 1\s*for \(uint32_t it = 0; it < max_iter; \+\+it\)", body)
    assert "return false;" in body


def test_polls_only_inside_bounded_helpers():
    polls = ("mbarrier.try_wait", "mbarrier.test_wait", "ld.acquire")
    for p in SOURCES:
        text = _strip_comments(p.read_text())
        if p == HELPERS:
            allowed = "".join(_function_body(text, n)[1] for n in BOUNDED + ("ld_acquire_u64",))
            for poll in polls:
                assert text.count(poll) == allowed.count(poll), (p.name, poll)
        else:
            for poll in polls:
                assert poll not in text, (p.name, poll)
    # the flag load itself is called only from the bounded poll
    for p in SOURCES:
        text = _strip_comments(p.read_text())
        uses = len(re.findall(r"\bld_acquire_u64\s*\(", text))
        if p == HELPERS:
            _, body = _function_body(text, "wait_flag_ge")
            assert uses == 2 and "ld_acquire_u64(" in body, uses  # definition + one call
        else:
            assert uses == 0, p.name


def test_every_wait_call_passes_a_limit():
    call = re.compile(r"\b(%s)\s*\(" % "|".join(BOUNDED))
    for p in SOURCES:
        text = _strip_comments(p.read_text())
        for m in call.finditer(text):
            depth, j = 0, m.end() - 1
            while True:
                depth += {"(": 1, ")": -1}.get(text[j], 0)
                if depth == 0:
                    break
                j += 1
            args = text[m.end():j]
            n_args = 1 + len(re.findall(r",(?![^()]*\))", args))
            assert n_args == 3, (p.name, text[m.start():j + 1])


def test_no_unconditional_loops():
    loop = re.compile(r"while\s*\(\s*(true|1)\s*\)|for\s*\(\s*;\s*;\s*\)")
    for p in SOURCES:
        assert not loop.search(_strip_comments(p.read_text())), p.name


def test_no_forced_kernel_stop():
    for p in SOURCES:
        text = _strip_comments(p.read_text())
        assert "__trap" not in text, p.name
        assert not re.search(r"\btrap\s*;", text), p.name
        assert not re.search(r"(?<![_a-z])assert\s*\(", text), p.name

