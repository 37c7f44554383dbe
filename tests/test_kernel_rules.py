"""Source rules of the CUDA kernels, checked on the text (no GPU):

* every loop that polls an mbarrier is bounded by a %globaltimer limit, so a
  wait that nothing completes ends with an error status instead of hanging;
* no device code traps or asserts (a failure is reported through the device
  error word and the context stays usable);
* every TMEM allocation in a kernel has a matching release in that kernel;
* no TMA or bulk copy uses cluster multicast (each CTA loads its own tiles;
  only tcgen05.commit arrivals are multicast across a CTA pair).
"""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_outlier_gemm_b200", "csrc")
SOURCES = sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def _text(name):
    src = open(os.path.join(CSRC, name)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def _loops(src):
    """(header, body) of every while / for loop, the body found by brace matching."""
    for m in re.finditer(r"\b(while|for)\s*\(", src):
        i, depth = m.end(), 1
        while depth:                       # the loop header's parentheses
            depth += {"(": 1, ")": -1}.get(src[i], 0)
            i += 1
        header = src[m.start():i]
        j = i
        while src[j].isspace():
            j += 1
        if src[j] != "{":                  # single-statement body
            k = src.index(";", j)
            yield header, src[j:k + 1]
            continue
        k, depth = j + 1, 1
        while depth:
            depth += {"{": 1, "}": -1}.get(src[k], 0)
            k += 1
        yield header, src[j:k]


def test_sources_found():
    assert {"act_quant.cu", "gemm_w4a4.cu", "gemm_int4.cu", "ptx.cuh"} <= set(SOURCES)


@pytest.mark.parametrize("name", SOURCES)
def test_every_barrier_poll_is_time_bounded(name):
    src = _text(name)
    polls = [(h, b) for h, b in _loops(src) if "try_wait" in h + b]
    for header, body in polls:
        assert "globaltimer" in header + body, f"{name}: unbounded poll {header.strip()}"
        assert re.search(r"return\s+false|break", body), f"{name}: poll without an exit {header.strip()}"


def test_the_poll_check_sees_the_waits_and_rejects_an_unbounded_one():
    found = sum(1 for n in SOURCES for h, b in _loops(_text(n)) if "try_wait" in h + b)
    assert found >= 4      # the bounded slow path and each kernel's drain wait
    planted = "void f(uint64_t* bar) {\n  while (!mbar_try_wait(bar, 0)) {\n  }\n}\n"
    (header, body), = [(h, b) for h, b in _loops(planted)]
    assert "try_wait" in header and "globaltimer" not in header + body


@pytest.mark.parametrize("name", SOURCES)
def test_no_traps_or_device_asserts(name):
    src = _text(name)
    assert "__trap" not in src and not re.search(r"\btrap\s*;", src)
    assert not re.search(r"(?<!static_)\bassert\s*\(", src)
    assert "__brkpt" not in src


@pytest.mark.parametrize("name", [s for s in SOURCES if s.endswith(".cu")])
def test_tmem_allocations_are_released(name):
    src = _text(name)
    allocs = len(re.findall(r"\btmem_alloc\w*\s*\(", src))
    frees = len(re.findall(r"\btmem_dealloc\w*\s*\(", src))
    assert allocs == frees


def _multicast_copies(src):
    return [line.strip() for line in src.splitlines() if "cp.async.bulk" in line and "multicast" in line]


@pytest.mark.parametrize("name", SOURCES)
def test_no_multicast_copies(name):
    assert _multicast_copies(open(os.path.join(CSRC, name)).read()) == []


def test_the_multicast_check_sees_a_planted_one():
    planted = ('asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes'
               '.multicast::cluster [%0], [%1, {%2, %3}], [%4], %5;" :: ...);\n'
               'asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64");')
    assert len(_multicast_copies(planted)) == 1
