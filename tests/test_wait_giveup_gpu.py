"""The kernels' bounded waits give up instead of hanging, and the step's
status word reports it (gad_attn_step_status, gad_oproj_status).

A stalled pipeline cannot be produced safely on purpose, so the test uses a
build of the library in which every pipeline wait gives up as soon as its
phase has not completed at the first, non-blocking probe (the production
limit is 2 s): a wait for a tensor-core result or a copy issued just before
never has, so every kernel with such waits gives up on every run.  The kernels
then take their give-up path for real: the waiting warps stop, the work in
flight (copies, tensor-core operations) is waited for, tensor memory is
freed, the status bit is set, and the step returns.  The steps run in a child
process that loads only that build; the test checks the bits, that the
process ends on its own, and that a later step in the same context is
correct.  The production library's status words read 0 after normal steps.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from paged_fp8_gated_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ATTN, OPROJ = 1, 2  # GAD_STATUS_ATTN_WAIT, GAD_STATUS_OPROJ_WAIT


def test_status_is_zero_after_normal_steps(cuda_dev):
    from paged_fp8_gated_b200 import binding
    for spec in (W.Spec("st_verify", B=3, L=8, seq_lens=[100, 2000, 5000], seed=511),
                 W.Spec("st_prefill", B=2, L=40, seq_lens=[0, 900], window=256, use_rope=True, seed=512)):
        inp = W.make_inputs(spec)
        ws = binding.alloc_workspace(inp["B"], inp["L"])
        ws.fill_(0xFF)                               # the step's first kernel clears the word
        H.run_gpu(inp, workspace=ws)
        assert binding.step_status(ws) == 0, spec.name
    x = W.oproj_input(32, seed=513).to("cuda")
    binding.oproj(x, W.oproj_weight().to("cuda"))
    assert binding.oproj_status() == 0


def test_waits_give_up_and_report(cuda_dev):
    from paged_fp8_gated_b200 import build
    build.build_short_wait()
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "giveup_child.py")], cwd=ROOT,
                          capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-3000:]
    res = json.loads(proc.stdout.strip().splitlines()[-1])
    assert res["verify"] & ATTN, res
    assert res["prefill"] & ATTN, res
    assert res["decode_oproj"] & OPROJ, res
    assert res["oproj"] & OPROJ and res["oproj_after_read"] == 0, res
    assert res["after_status"] == 0 and res["after_ok"], res
