"""The activation parameters the pages print, and the workloads built on them."""
import json
import math
import os

import numpy as np

from oracle import layer as L
from workloads.synth import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "activation_params.json")


def test_oai_workload_uses_printed_parameters():
    p = json.load(open(GOLDEN))["oai_swiglu_example_model"]
    wl = WORKLOADS["oai"]
    assert (wl.alpha, wl.up_bias, wl.limit) == (p["activation_alpha"], p["activation_up_bias"],
                                                 p["activation_clamp"])


def test_printed_defaults_give_standard_swiglu():
    d = json.load(open(GOLDEN))["defaults_standard_swiglu"]
    g = np.linspace(-20, 20, 401)
    u = np.linspace(3, -3, 401)
    a = L.swiglu(g, u, d["activation_alpha"], d["activation_up_bias"], math.inf)
    for wl in (WORKLOADS["tiny"], WORKLOADS["decode"], WORKLOADS["prefill"], WORKLOADS["mxfp4"]):
        assert (wl.alpha, wl.up_bias) == (d["activation_alpha"], d["activation_up_bias"])
        np.testing.assert_array_equal(L.swiglu(g, u, wl.alpha, wl.up_bias, wl.limit), a)
