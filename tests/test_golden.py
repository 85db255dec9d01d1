"""The oracle still reproduces the stored expectations for the tiny workload."""
import json
import os

import numpy as np

from tests.golden.make_golden import tiny_expectations

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_pipeline_golden():
    with open(os.path.join(HERE, "tiny_pipeline.json")) as f:
        stored = json.load(f)
    now = tiny_expectations()
    assert stored.keys() == now.keys()
    for k in stored:
        if isinstance(stored[k], list) and stored[k] and isinstance(stored[k][0], float):
            np.testing.assert_array_equal(np.array(stored[k]), np.array(now[k]), err_msg=k)
        else:
            assert stored[k] == now[k], k
