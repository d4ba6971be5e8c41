"""DraftCycle (the graph-replayed cycle with host copies) against the
individual C-ABI calls and the oracle's verification, on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wi", [0, 1, 2])
def test_cycle_matches_separate_calls(wi):
    import block_draft_selection_b200 as bds
    w = syn.workload(wi)
    H, W = syn.hidden(w), syn.lm_head(w)
    E, M = syn.selector_tables(w)
    x, prev = syn.conv_input(w)
    a0, a1 = syn.conv_taps(w)
    W_d, E_d, M_d, a0_d, a1_d = dev_bf16(W), dev_bf16(E), dev_bf16(M), dev_bf16(a0), dev_bf16(a1)
    # target tokens from the library's own head on the noised states (fine for a self-consistency check)
    _, tix, _ = bds.dflash_lmhead_topk(dev_bf16(syn.target_hidden(w, H)), W_d)
    target = tix[:, 0].contiguous().view(w.B, w.L + 1)

    cyc = bds.DraftCycle(W_d, E_d, M_d, a0_d, a1_d, w.B, w.L, w.P)
    cyc.host_in["H"].copy_(bds.bf16_tensor(H, None))
    cyc.host_in["x"].copy_(bds.bf16_tensor(x, None))
    cyc.host_in["prev"].copy_(bds.bf16_tensor(prev, None))
    cyc.host_in["target"].copy_(target.cpu())
    out = {k: v.clone() for k, v in cyc.run().items()}
    out2 = cyc.run()                       # a second replay gives the same results
    for k in out:
        assert torch.equal(out[k], out2[k]), k
    assert int(cyc.status.item()) == 0

    y = bds.dflash_conv2tap(dev_bf16(x), a0_d, a1_d, dev_bf16(prev))
    lp, ix, _ = bds.dflash_lmhead_topk(dev_bf16(H), W_d)
    tok, slot, score, _ = bds.dflash_path_select(lp, ix, E_d, M_d, w.B, w.L)
    torch.cuda.synchronize()
    assert torch.equal(out["y"], y.cpu())
    assert torch.equal(out["path_tok"], tok.cpu())
    racc, rnxt = oracle.verify(tok.cpu().numpy(), target.cpu().numpy())
    np.testing.assert_array_equal(out["accept_len"].numpy(), racc)
    np.testing.assert_array_equal(out["next_token"].numpy(), rnxt)


@pytest.mark.parametrize("wi", [1, 2])
def test_pipeline_steps_match_sequential_cycle(wi):
    """DraftPipeline (two cycles stepped alternately on two streams) returns,
    for every step, the results a sequential DraftCycle gives on the same
    inputs: six steps whose hidden states and conv inputs differ."""
    import block_draft_selection_b200 as bds
    w = syn.workload(wi)
    W = syn.lm_head(w)
    E, M = syn.selector_tables(w)
    a0, a1 = syn.conv_taps(w)
    W_d, E_d, M_d, a0_d, a1_d = dev_bf16(W), dev_bf16(E), dev_bf16(M), dev_bf16(a0), dev_bf16(a1)
    steps = []
    for s in range(6):
        ws = syn.Workload(w.name, B=w.B, L=w.L, P=w.P, d=w.d, V=w.V, r=w.r, sigma=w.sigma, seed=w.seed + 100 + s)
        H = syn.hidden(ws)
        x, prev = syn.conv_input(ws)
        _, tix, _ = bds.dflash_lmhead_topk(dev_bf16(syn.target_hidden(ws, H)), W_d)
        steps.append({"H": bds.bf16_tensor(H, None), "x": bds.bf16_tensor(x, None),
                      "prev": bds.bf16_tensor(prev, None), "target": tix[:, 0].contiguous().view(w.B, w.L + 1).cpu()})
    seq = bds.DraftCycle(W_d, E_d, M_d, a0_d, a1_d, w.B, w.L, w.P)
    ref = []
    for inp in steps:
        for k, v in inp.items():
            seq.host_in[k].copy_(v)
        ref.append({k: v.clone() for k, v in seq.run().items()})
    pipe = bds.DraftPipeline(W_d, E_d, M_d, a0_d, a1_d, w.B, w.L, w.P)
    got = []
    for inp in steps:
        hin, prev_out = pipe.host_in()
        if prev_out is not None:
            got.append({k: v.clone() for k, v in prev_out.items()})
        for k, v in inp.items():
            hin[k].copy_(v)
        pipe.launch()
    got += [{k: v.clone() for k, v in o.items()} for o in pipe.drain()]
    assert len(got) == len(ref)
    for i, (g, r) in enumerate(zip(got, ref)):
        for k in r:
            assert torch.equal(g[k], r[k]), (i, k)
