"""The planner's cost model against the device: predicted and measured iteration times.

NanoFlow searches the nano-batch configuration taking into account how concurrent operations slow
one another (arXiv abstract). After nf_calibrate (per-kernel rates, decode bandwidth at five SM
shares, co-run slow-downs at three attention shares), the planner's best plan for each template
and nano-batch count is run on the batch and timed in steady state (each plan alone for half a second
first); the prediction error of each is printed, and the plan the model ranks first must be within
10% of the fastest one measured, every prediction within 20%.
"""
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CANDIDATES = [dict(nano=1, template=0), dict(nano=1, template=2), dict(nano=2, template=1),
              dict(nano=2, template=2), dict(nano=3, template=1), dict(nano=4, template=2)]


def _time_us(dw, plan, reps):
    # steady state: the GPU runs at its power cap, and a short run would inherit the clock the previous
    # plan left, so each plan runs alone for about half a second before it is timed
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 0.5:
        for _ in range(4):
            dw.forward(plan)
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        dw.forward(plan)
    e1.record()
    torch.cuda.synchronize()
    assert dw.sync() == 0
    return e0.elapsed_time(e1) * 1000.0 / reps


@pytest.mark.parametrize("name,reps", [("llama3_8b_layer", 20), ("llama2_70b_slice", 3)])
def test_predicted_and_measured_plan_times(name, reps):
    from intra_device_overlapped_b200.harness import DeviceWorkload
    from synth.workloads import WORKLOADS
    dw = DeviceWorkload(WORKLOADS[name], DEV, keep_logits=False)
    try:
        cost = dw.calibrate()
        print(f"{name} cost model: " + ", ".join(f"{k}={v}" for k, v in cost.items()))
        rows = []
        for opts in CANDIDATES:
            plan = dw.plan(**opts)
            meas = _time_us(dw, plan, reps)
            rows.append((plan.describe(), plan.predicted_us, meas))
        errs = []
        for desc, pred, meas in rows:
            err = (pred - meas) / meas
            errs.append(abs(err))
            print(f"{name}: predicted {pred:9.1f} us, measured {meas:9.1f} us, error {100 * err:+6.1f}%  "
                  f"n={desc['n_nano']} {desc['template']} sm_attn={desc['sm_attn']} order={desc['order']}")
        print(f"{name}: largest prediction error {100 * max(errs):.1f}%, mean {100 * float(np.mean(errs)):.1f}%")
        best_pred = min(rows, key=lambda r: r[1])
        best_meas = min(rows, key=lambda r: r[2])
        # the model's first choice runs within 10% of the best measured candidate
        assert best_pred[2] <= 1.10 * best_meas[2], (best_pred, best_meas)
        assert max(errs) < 0.2
    finally:
        dw.close()
