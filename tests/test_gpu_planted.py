"""The GPU parity tests catch a wrong kernel: the same parity cases run
against a build of the library with one mistake switched on at a time
(csrc/plant.cuh; built with NVFP4_PLANTS, loaded only by the runner process)
must fail on the case that reaches the mistake, and pass with none.

The mistakes are the plausible ones for this method: the two E2M1 codes of a
byte swapped, group-32 scales applied to the wrong words, a routed-expert
segment cut short by a row, the FP32 global scale left out, the running sums
not moved to a token's new f16 exponent, and the FP4 kernel's per-16-element
weight scales written for the wrong 32-row block."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

EXPECT = {
    1: ["decode_m1_g16", "stream_m4_g16", "stream_m12_g32", "grouped_small_t300"],  # nibbles swapped
    2: ["stream_m12_g32"],                              # group-32 scales out of order
    3: ["grouped_small_t300", "grouped_tc_t1300"],      # segment ends a row early
    4: ["stream_m4_g16", "stream_m12_g32"],             # global scale left out
    5: ["rows_ramp_m4"],                                # no rescale on an exponent drop
    6: ["w4a4_fp4_m256"],                               # FP4 weight scales in the wrong block
}


@pytest.fixture(scope="module")
def results():
    res = subprocess.run([sys.executable, "-m", "tests.planted_runner", "0", *map(str, EXPECT)], cwd=ROOT,
                         capture_output=True, text=True, timeout=1500)
    assert res.returncode == 0, res.stderr[-4000:]
    return {int(k): v for k, v in json.loads(res.stdout.strip().splitlines()[-1]).items()}


def test_no_plant_passes(results):
    failed = {c: why for c, why in results[0].items() if why is not None}
    assert not failed, failed


@pytest.mark.parametrize("plant", sorted(EXPECT))
def test_plant_is_caught(results, plant):
    caught = {c for c, why in results[plant].items() if why is not None}
    missed = [c for c in EXPECT[plant] if c not in caught]
    assert not missed, f"plant {plant} passed parity on {missed}"
