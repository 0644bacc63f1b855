"""Host logic of the reverse traversal's schedule (csrc/bptt_plan.h, the
header rlt_backward's driver runs), checked without a GPU.

tests/bw_plan_check.cpp replays the schedule for chunks of 1..257 steps,
start positions 0..1000 and windows 1..129. The schedule has three parts:
groups and batches, the SWA terms added directly, and the ranges formed from
saved records. The checker asserts that every SWA term reaches its key's
gradient exactly once, before the gradient is read, from a record that still
holds its step. It also asserts that the batches and the group column blocks
line up. Shifted variants show that the checks bite:
  * a direct bound one lower double-counts terms;
  * a direct bound one higher loses them;
  * W - 2 record slots (one below the W - 1 the records need) read
    overwritten records.
"""
import os
import re
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "token_recurrent_decoding_b200", "csrc")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("bwplan") / "bw_plan_check")
    subprocess.check_call([gxx, "-O2", "-std=c++17", "-I", CSRC,
                           os.path.join(HERE, "bw_plan_check.cpp"), "-o", exe])
    return exe


def _run(exe, direct_shift=0, slot_shift=0):
    out = subprocess.run([exe, str(direct_shift), str(slot_shift)], capture_output=True,
                         text=True, check=True).stdout
    m = re.search(r"cases (\d+) failing (\d+)", out)
    assert m, out
    return int(m.group(1)), int(m.group(2)), out


def test_schedule_invariants_hold(checker):
    cases, failing, out = _run(checker)
    assert cases == 14 * 5 * 10
    assert failing == 0, out


# record_slots(W) = RECOMP + W; a shift of -(RECOMP + 2) leaves W - 2 slots
@pytest.mark.parametrize("direct_shift,slot_shift", [(-1, 0), (1, 0), (0, -10)])
def test_planted_schedule_mistakes_are_caught(checker, direct_shift, slot_shift):
    cases, failing, _ = _run(checker, direct_shift, slot_shift)
    assert failing > 0


def test_records_need_exactly_w_minus_one_slots(checker):
    """W - 1 slots suffice (shift -(RECOMP + 1)); the margin is RECOMP + 1."""
    cases, failing, out = _run(checker, 0, -9)
    assert failing == 0, out
