"""The bench's further rows run end to end on the GPU (a few steps each) and
produce a complete JSON line (needs a B200)."""
import argparse
import json

import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("row", ["moving", "qknorm", "window", "ulysses"])
def test_row_runs_and_reports(row):
    args = argparse.Namespace(steps=3, warmup=3, row=row, config=3)
    line = bench.run_row(args, 0, 1, 0, torch.device("cuda", 0), None)
    json.dumps(line)
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["gpu_launches"] > 0
    roof = line["roofline"]
    assert roof["achieved"] > 0 and 0 < roof["frac"] < 2
    assert line["config"]["row"] == row
