"""Performance floor (regression alarm): each shape of the offline schedule sweep
(sm_gemm_b200/tune.py) must run within 1.5x of the time recorded when its schedule was
chosen (sm_gemm_b200/tuned_configs.json). The margin absorbs box-to-box and clock
differences; what it catches is a change that makes a kernel markedly slower (a register
spill, an instruction-cache blow-up, a lost pipeline overlap), in the spirit of the
regression checks of the DeepGEMM kernel-library walkthrough (zwxr.cn), section 5.2.
The shape runs with the default schedule, i.e. the table's choice compiled into the
library."""
import json
import os

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RECORD = os.path.join(ROOT, "sm_gemm_b200", "tuned_configs.json")


def _shapes():
    if not os.path.exists(RECORD):
        return []
    return sorted(json.load(open(RECORD))["shapes"].items())


@pytest.mark.parametrize("name,rec", _shapes() or [pytest.param(None, None, marks=pytest.mark.skip("no sweep record"))])
def test_tuned_shape_meets_floor(cuda_device, name, rec):
    import torch
    import sm_gemm_b200 as sg
    from sm_gemm_b200 import tune
    for v in ("SMGEMM_GROUP_M", "SMGEMM_SPLITK", "SMGEMM_SCHED", "SMGEMM_FORCE_CONFIG", "SMGEMM_PAIR"):
        assert v not in os.environ, f"{v} is set: the floor is for the default schedule"
    us = tune.time_shape(sg, torch, rec["kind"], rec["M"], rec["N"], rec["K"], rec["layout_a"], rec["layout_b"])
    plan = sg.last_config()
    assert us <= 1.5 * rec["us"], f"{name}: {us:.1f} us against {rec['us']:.1f} us recorded ({plan})"
