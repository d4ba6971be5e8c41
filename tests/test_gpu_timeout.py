"""The LM-head kernel's bounded waits, made to run out on purpose (no fault:
every wait gives up at its deadline, records DFLASH_ERR_TIMEOUT in the
caller's status word, drains what it has in flight and returns).

Weight-streaming orientation only (the qwen3-4b-bs1 shape, M = 7: one CTA
per SM, no 2-CTA pairs).  A child process sets DFLASH_TIMEOUT_NS, which the
library reads at every call, to a budget far below the call's running time --
once so small that the first copies cannot land in time and once so that the
waits run out in the middle of the weight stream -- then clears it: the
status must say "timed out" both times, every call must return, and the
normal calls that follow in the same process must still match the oracle."""
import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

pytestmark = pytest.mark.gpu

BUDGETS_NS = (2_000, 40_000)     # the full call takes about 140 us


def child():
    sys.path[:0] = [ROOT, HERE]
    import numpy as np
    import torch

    import block_draft_selection_b200 as bds
    import block_draft_synth as syn
    import oracle
    from helpers import dev_bf16

    w = syn.workload("qwen3-4b-bs1")
    H, W = syn.hidden(w), syn.lm_head(w)
    Hd, Wd = dev_bf16(H), dev_bf16(W)
    ws = bds.workspace(w.M, w.V, w.d, "cuda")

    def call():
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        lp, ix, lse = bds.dflash_lmhead_topk(Hd, Wd, ws=ws, dev_status=status)
        torch.cuda.synchronize()
        return int(status.item()), lp, ix

    codes = []
    for budget in BUDGETS_NS:
        os.environ["DFLASH_TIMEOUT_NS"] = str(budget)
        codes.append(call()[0])
        del os.environ["DFLASH_TIMEOUT_NS"]
        code, lp, ix = call()               # the next normal call in the same process
        codes.append(code)
    rlp, rix, rlse, z = oracle.lmhead_topk(H, W, 16, return_logits=True)
    lp_np, ix_np = lp.cpu().numpy(), ix.cpu().numpy()
    bad = []
    for m in range(w.M):
        ok, msg = oracle.topk_margin_ok(z[m], rlse[m], ix_np[m], lp_np[m])
        if not ok:
            bad.append(f"row {m}: {msg}")
    print(json.dumps({"codes": codes, "bad": bad, "timeout_code": bds.DFLASH_ERR_TIMEOUT}), flush=True)


def test_wait_budget_runs_out_and_context_survives():
    out = subprocess.run([sys.executable, os.path.abspath(__file__), "--child"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    T = d["timeout_code"]
    assert d["codes"] == [T, 0, T, 0], d["codes"]
    assert not d["bad"], d["bad"]


if __name__ == "__main__" and "--child" in sys.argv:
    child()
