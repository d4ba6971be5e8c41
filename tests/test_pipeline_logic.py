"""DraftPipeline's host-side sequencing on the CPU, with stand-in cycles (no
GPU): step i runs on cycle i % 2; host_in() hands back that cycle's previous
step's results before the caller refills its inputs; drain() returns the
steps still in flight oldest first; launching a cycle whose last step was
not collected is refused."""
import pytest

import block_draft_selection_b200.cycle as cyc


class FakeCycle:
    def __init__(self, log, name):
        self.log, self.name = log, name
        self.host_in = {"step": None}
        self._launched = None

    def launch(self, stream):
        assert self._launched is None, "launched twice without wait"
        self._launched = self.host_in["step"]
        self.log.append(("launch", self.name, self._launched, stream))

    def wait(self):
        assert self._launched is not None, "wait without launch"
        out, self._launched = {"step": self._launched}, None
        self.log.append(("wait", self.name, out["step"]))
        return out


@pytest.fixture
def pipe(monkeypatch):
    log = []
    p = cyc.DraftPipeline.__new__(cyc.DraftPipeline)
    p.cycles = [FakeCycle(log, 0), FakeCycle(log, 1)]
    p.streams = ["s0", "s1"]
    p._pending = [False, False]
    p._i = 0
    p.log = log
    return p


def test_results_come_back_in_step_order(pipe):
    got = []
    for step in range(7):
        hin, prev = pipe.host_in()
        if prev is not None:
            got.append(prev["step"])
        hin["step"] = step
        pipe.launch()
    got += [o["step"] for o in pipe.drain()]
    assert got == list(range(7))
    launches = [(e[1], e[2], e[3]) for e in pipe.log if e[0] == "launch"]
    assert launches == [(i % 2, i, f"s{i % 2}") for i in range(7)]
    # a cycle's previous step is collected before its inputs are refilled
    for i, e in enumerate(pipe.log):
        if e[0] == "launch" and e[2] >= 2:
            assert ("wait", e[1], e[2] - 2) in pipe.log[:i]


def test_launch_needs_host_in_first(pipe):
    for step in range(2):
        hin, _ = pipe.host_in()
        hin["step"] = step
        pipe.launch()
    with pytest.raises(RuntimeError):
        pipe.launch()          # cycle 0 still holds step 0's results
    assert [o["step"] for o in pipe.drain()] == [0, 1]
    assert pipe.drain() == []
