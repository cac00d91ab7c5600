"""The device status word of the prefill: a bounded wait that runs out is
reported to the caller instead of leaving wrong outputs behind silently.

The failure is made safely: the debugging knob tells the sequential kernel's
copy producer to issue nothing, so its consumers' first wait on a chunk record
runs out while no copy, TMA load or MMA is in flight. The kernels then return
early, the status word holds the waiting side's code, and the context stays
usable for the next call.
"""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

import oracle
from common import rel_l2, to_cuda
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu

KDA_OK, KDA_ERR_DEVICE_STATUS = 0, 6
ERR_FULL = 1  # code of the sequential kernel's wait for a chunk record
# Poll limit for the starved run: far above any wait of a working pipeline,
# small enough that the starved wait ends within milliseconds.
SHORT_LIMIT = 20000

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _problem():
    return I.make_prefill(1, 200, 2, 128, torch.bfloat16, gate_shift=-1.0, s0_std=0.05,
                          seed=71)


def test_status_is_ok_after_a_normal_call():
    g = to_cuda(_problem())
    call = kda.ChunkFwdCall(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"],
                            algo="tcgen05")
    call.run()
    assert kda.kda_chunk_fwd_status(call.workspace) == (KDA_OK, 0)


def test_starved_carry_reports_its_wait_and_the_next_call_is_clean():
    x = _problem()
    g = to_cuda(x)
    call = kda.ChunkFwdCall(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"],
                            algo="tcgen05")
    try:
        kda.kda_debug_set_wait_limit(SHORT_LIMIT, starve_carry=True)
        call.run()
        st, code = kda.kda_chunk_fwd_status(call.workspace)
    finally:
        kda.kda_debug_set_wait_limit(0, starve_carry=False)
    assert st == KDA_ERR_DEVICE_STATUS
    assert code == ERR_FULL
    # the same workspace and context: the next call is clean and correct
    o, S = call.run()
    assert kda.kda_chunk_fwd_status(call.workspace) == (KDA_OK, 0)
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                                  None, x["scale"])
    assert rel_l2(o, o_ref) <= 2e-2 and rel_l2(S, S_ref) <= 2e-2


def test_debug_sync_returns_the_device_status():
    """With KDA_DEBUG_SYNC=1 the prefill call itself waits and returns
    KDA_ERR_DEVICE_STATUS (a fresh process, since the setting is read once)."""
    script = textwrap.dedent(f"""
        import sys, torch
        sys.path.insert(0, {ROOT!r})
        from gated_delta_rule_132_b200 import inputs as I, kda
        x = I.make_prefill(1, 200, 2, 128, torch.bfloat16, -1.0, 0.05, seed=71, device="cuda")
        a = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
        kda.kda_chunk_fwd(*a, algo="tcgen05")          # clean call: no error
        kda.kda_debug_set_wait_limit({SHORT_LIMIT}, starve_carry=True)
        try:
            kda.kda_chunk_fwd(*a, algo="tcgen05")
        except kda.KdaError as e:
            print("STATUS", e.status)
        finally:
            kda.kda_debug_set_wait_limit(0, starve_carry=False)
        kda.kda_chunk_fwd(*a, algo="tcgen05")          # clean again
        print("CLEAN")
    """)
    env = dict(os.environ, KDA_DEBUG_SYNC="1")
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert f"STATUS {KDA_ERR_DEVICE_STATUS}" in r.stdout and "CLEAN" in r.stdout
