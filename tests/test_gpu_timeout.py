"""The LM-head kernel's bounded waits, made to run out on purpose (no fault:
every wait gives up at its deadline, records DFLASH_ERR_TIMEOUT in the
caller's status word, drains what it has in flight and returns).

A child process sets DFLASH_TIMEOUT_NS, which the library reads at every
call, to a budget far below the call's running time -- once so small that
the first copies cannot land in time and once so that the waits run out in
the middle of the weight stream -- then clears it.  The status must say
"timed out" both times, every call must return, and the normal calls that
follow in the same process must still match the oracle.  Three paths:
- weight streaming (qwen3-4b-bs1, M = 7): one CTA per SM;
- tensor-bound on 2-CTA pairs (qwen3-4b-batched, M = 448): the pair's
  loads all complete on the leader's barriers, so on giving up the leader
  drains both CTAs' copies (the other CTA hands over its count of loads);
- tensor-bound on single CTAs (the same shape with DFLASH_PAIR=0)."""
import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

pytestmark = pytest.mark.gpu

# (workload, extra environment, budgets in ns: far below the call's time)
CASES = [("qwen3-4b-bs1", {}, (2_000, 40_000)),            # call: about 140 us
         ("qwen3-4b-batched", {}, (2_000, 100_000)),        # call: about 360 us
         ("qwen3-4b-batched", {"DFLASH_PAIR": "0"}, (2_000, 100_000))]


def child(case):
    sys.path[:0] = [ROOT, HERE]
    import numpy as np
    import torch

    import block_draft_selection_b200 as bds
    import block_draft_synth as syn
    import oracle
    from helpers import dev_bf16

    name, env, budgets = CASES[case]
    os.environ.update(env)
    w = syn.workload(name)
    H, W = syn.hidden(w), syn.lm_head(w)
    Hd, Wd = dev_bf16(H), dev_bf16(W)
    ws = bds.workspace(w.M, w.V, w.d, "cuda")

    def call():
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        lp, ix, lse = bds.dflash_lmhead_topk(Hd, Wd, ws=ws, dev_status=status)
        torch.cuda.synchronize()
        return int(status.item()), lp, ix

    codes = []
    for budget in budgets:
        os.environ["DFLASH_TIMEOUT_NS"] = str(budget)
        codes.append(call()[0])
        del os.environ["DFLASH_TIMEOUT_NS"]
        code, lp, ix = call()               # the next normal call in the same process
        codes.append(code)
    # the first and last row of every 128-row tile (every row when M <= 128)
    rows = sorted({r for t0 in range(0, w.M, 128) for r in (t0, min(w.M, t0 + 128) - 1)} | set(range(min(w.M, 8))))
    rlp, rix, rlse, z = oracle.lmhead_topk(H[rows], W, 16, return_logits=True)
    lp_np, ix_np = lp.cpu().numpy(), ix.cpu().numpy()
    bad = []
    for n, m in enumerate(rows):
        ok, msg = oracle.topk_margin_ok(z[n], rlse[n], ix_np[m], lp_np[m])
        if not ok:
            bad.append(f"row {m}: {msg}")
    print(json.dumps({"codes": codes, "bad": bad, "timeout_code": bds.DFLASH_ERR_TIMEOUT}), flush=True)


@pytest.mark.parametrize("case", range(len(CASES)), ids=[c[0] + ("-single-cta" if c[1] else "") for c in CASES])
def test_wait_budget_runs_out_and_context_survives(case):
    out = subprocess.run([sys.executable, os.path.abspath(__file__), "--child", str(case)], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    T = d["timeout_code"]
    assert d["codes"] == [T, 0, T, 0], d["codes"]
    assert not d["bad"], d["bad"]


if __name__ == "__main__" and "--child" in sys.argv:
    child(int(sys.argv[sys.argv.index("--child") + 1]))
