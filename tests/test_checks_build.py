"""The checking build (liblatentmoe_checks.so, LMOE_CHECKS=1) on the GPU.

Every index a kernel reads from memory (tile records, permutation and slot
indices, flag and z element lists) is bounds-checked on the device; a failed
check records LMOE_ERR_INVALID_ARG and the access is skipped. This stands in
for a memory checker: the parity cases must pass with no check failing, and one
planted out-of-range index must be caught and reported. Each case runs in a
child process that loads the checking build (LATENTMOE_CHECKS=1).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("case", ["layer", "ep", "nvfp4", "corrupt_slot"])
def test_checking_build(case):
    env = dict(os.environ, LATENTMOE_CHECKS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checks_child.py"), case], env=env,
                       stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True, timeout=900)
    print(r.stdout[-3000:])
    assert r.returncode == 0, r.stdout[-3000:]
    assert "case %s ok" % case in r.stdout
