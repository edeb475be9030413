"""Static checks of the CUDA sources (no GPU): constructs that the library must not contain.

* No TMA or bulk copy with cluster multicast: every load of the library reads this GPU's own
  memory and is issued per CTA, so none needs it, and the build keeps it out altogether.
* No batched memcpy entry point of the CUDA runtime or driver: the library issues no host copies
  at all, and those calls have faulted GPUs of this model with this driver.
* No device trap or assert: failures are reported through status words and bounded waits.
* Every `mbarrier.try_wait` loop sits in a function that also reads the global timer (bounded).
"""
from __future__ import annotations

import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCES = sorted(glob.glob(os.path.join(ROOT, "xlstm_mlstm_cell_b200", "csrc", "*.cu")) +
                 glob.glob(os.path.join(ROOT, "xlstm_mlstm_cell_b200", "csrc", "*.cuh")) +
                 glob.glob(os.path.join(ROOT, "xlstm_mlstm_cell_b200", "csrc", "*.h")) +
                 glob.glob(os.path.join(ROOT, "include", "*.h")))


def _text(path):
    return open(path).read()


def test_sources_found():
    names = {os.path.basename(p) for p in SOURCES}
    assert {"fwd_tc.cu", "step.cu", "slstm.cu", "tc_common.cuh", "mlstm.h", "slstm.h"} <= names


def test_no_cluster_multicast():
    for p in SOURCES:
        assert ".multicast::cluster" not in _text(p), p


def test_no_batched_memcpy():
    pat = re.compile(r"(cuda|cu)Memcpy(3D)?Batch")
    for p in SOURCES:
        assert not pat.search(_text(p)), p


def test_no_device_trap_or_assert():
    pat = re.compile(r"__trap\s*\(|\bassert\s*\(|\btrap;")
    for p in SOURCES:
        assert not pat.search(_text(p)), p


def test_mbarrier_waits_are_bounded():
    # each function body that polls an mbarrier also checks the global timer, or is the single
    # non-blocking probe that such a bounded loop calls
    for p in SOURCES:
        text = _text(p)
        for m in re.finditer(r"mbarrier\.try_wait", text):
            start = text.rfind("__device__", 0, m.start())
            start = max(start, text.rfind("MLSTM_DEVINL", 0, m.start()))
            end = text.find("\n}\n", m.start())
            body = text[start:end]
            probe = "return" in body and not re.search(r"\b(for|while)\s*\(", body)
            assert probe or "global_timer" in body, "%s: unbounded mbarrier wait near offset %d" % (p, m.start())


def test_callers_of_the_mbarrier_probe_are_bounded():
    # a loop around the non-blocking probe must sit in a function that reads the global timer
    for p in SOURCES:
        text = _text(p)
        for m in re.finditer(r"\b(while|for)\s*\([^;{]*mbar_try_wait|mbar_try_wait\([^)]*\)\)\s*return", text):
            start = text.rfind("__device__", 0, m.start())
            end = text.find("\n}\n", m.start())
            assert "global_timer" in text[start:end], "%s: unbounded loop on mbar_try_wait near %d" % (p, m.start())
