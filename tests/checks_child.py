"""Child process of test_checks_build.py: runs one case against the checking build
(LATENTMOE_CHECKS=1 makes the binding load liblatentmoe_checks.so)."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import latentmoe_layer_b200 as lm  # noqa: E402
import synth  # noqa: E402
import helpers as H  # noqa: E402

assert os.environ.get("LATENTMOE_CHECKS") == "1" and lm.LIB_PATH.endswith("liblatentmoe_checks.so"), lm.LIB_PATH


def case_layer():
    from test_layer_gpu import run_and_compare, RAGGED, RAGGED_X32, TINY, PAIRW
    # PAIRW: widths that make option 4 run 2-SM pair tiles (RAGGED's do not)
    for shape, mode, path in ((TINY, 0, 1), (RAGGED, 0, 1), (RAGGED, 0, 2), (RAGGED, 0, 3), (RAGGED, 0, 4),
                              (PAIRW, 0, 4), (RAGGED_X32, 0, 1), (RAGGED, 1, 0)):
        (ma, rf), layer = run_and_compare(shape, mode=mode, path=path)
        assert layer.stats().device_error == 0
        print("%s mode=%d path=%d max_abs=%.3g rel_fro=%.3g" % (shape.name, mode, path, ma, rf))


def case_ep():
    from test_ep_gpu import check_ep_against_oracle, RAGGED
    check_ep_against_oracle(RAGGED, 2, [0, 170, RAGGED.T])


def case_nvfp4():
    from test_nvfp4_gpu import run_nvfp4, RAGGED4
    layer, _, _, _ = run_nvfp4(RAGGED4)
    assert layer.stats().device_error == 0


def case_corrupt_slot():
    """An out-of-range row index planted in the workspace between the expert-parallel front
    and back stages: the combine's check refuses it (no access), the call's error word says
    LMOE_ERR_INVALID_ARG, and the next call on the handle reports it."""
    from test_ep_gpu import stages, RAGGED
    layer, dev = H.device_layer(RAGGED)
    send_rows, send_w, counts = stages(layer, dev["x"])
    o = torch.zeros((send_rows.shape[0], RAGGED.L), dtype=torch.float32, device="cuda")
    layer.ep_experts(send_rows, send_w, counts, 1, o)
    slot = layer.ws_view(layer.layout(RAGGED.T).slot, (RAGGED.T * RAGGED.k,), torch.int32)
    slot[5] = 1 << 30
    y = torch.empty((RAGGED.T, RAGGED.H), dtype=torch.float32, device="cuda")
    layer.ep_back(o, y)
    torch.cuda.synchronize()
    assert layer.stats().device_error == lm.LMOE_ERR_INVALID_ARG
    assert bool(torch.isfinite(y).all())
    try:
        layer.forward(dev["x"])
        raise AssertionError("the recorded error was not reported")
    except lm.LmoeError as e:
        assert e.status == lm.LMOE_ERR_INVALID_ARG
    y2 = layer.forward(dev["x"])  # reported once; the handle works again
    torch.cuda.synchronize()
    assert layer.stats().device_error == 0 and bool(torch.isfinite(y2).all())


if __name__ == "__main__":
    globals()["case_" + sys.argv[1]]()
    print("case %s ok" % sys.argv[1])
