"""The benchmark cycle's two-stream schedule, on the host with stand-in streams and events.

`Cycle.step` issues Sparse-to-Dense's chain on the caller's stream and Sparrow's chain (HSR
projection, text-anchored attention) on a second stream, joins them before verification, runs
the greedy rule on the second stream after verification and joins again at the end.  Each
chain must keep its order and every cross-stream edge must be in place, or a replayed graph
could read a draft before it is written.  No GPU: the streams and events only log what is
asked of them."""
import bench


class FakeEvent:
    def __init__(self, log, i):
        self.log, self.i = log, i

    def record(self, stream):
        self.log.append(("record", self.i, stream.name))


class FakeStream:
    def __init__(self, log, name):
        self.log, self.name = log, name

    def wait_event(self, ev):
        self.log.append(("wait", self.name, ev.i))


KINDS = ["topk", "stage"] + [k for t in range(3) for k in ("sparse", "hsr", "text_anchored")] + \
    ["verify", "accept_greedy", "accept_sample"]


def make_cycle(log):
    cyc = object.__new__(bench.Cycle)
    cyc.torch = None  # (only used to find the current stream when none is given)
    cyc.side = FakeStream(log, "side")
    cyc.events = [FakeEvent(log, i) for i in range(4)]
    cyc.calls = [(k, i, (lambda s, b, k=k: log.append(("call", k, s.name, b))))
                 for i, k in enumerate(KINDS)]
    return cyc


def test_two_stream_schedule():
    log = []
    cyc = make_cycle(log)
    main = FakeStream(log, "main")
    bench.Cycle.step(cyc, main, 1)
    calls = [(e[1], e[2]) for e in log if e[0] == "call"]
    assert [k for k, _ in calls] == KINDS  # every call once, in the cycle's order
    side = {"hsr", "text_anchored", "accept_greedy"}
    assert all(s == ("side" if k in side else "main") for k, s in calls)
    assert all(e[3] == 1 for e in log if e[0] == "call")  # the input set is passed on
    pos = {e: i for i, e in enumerate(log)}

    def at(kind):
        return next(i for i, e in enumerate(log) if e[0] == "call" and e[1] == kind)

    # fork: the side stream waits for the main stream's state at the start of the step
    assert log[0] == ("record", 0, "main") and log[1] == ("wait", "side", 0)
    # join before verification: the side stream's last text-anchored call is recorded first
    last_ta = max(i for i, e in enumerate(log) if e[0] == "call" and e[1] == "text_anchored")
    assert last_ta < pos[("record", 1, "side")] < pos[("wait", "main", 1)] < at("verify")
    # the greedy rule on the side stream only after verification
    assert at("verify") < pos[("record", 2, "main")] < pos[("wait", "side", 2)] < \
        at("accept_greedy")
    # the step ends with the main stream waiting for the side stream's last call
    assert log[-2:] == [("record", 3, "side"), ("wait", "main", 3)]
    assert at("accept_greedy") < len(log) - 2


def test_subset_of_kinds_stays_on_one_stream():
    log = []
    cyc = make_cycle(log)
    main = FakeStream(log, "main")
    bench.Cycle.step(cyc, main, 0, kinds=("hsr", "text_anchored", "verify"))
    assert all(e[0] == "call" and e[2] == "main" for e in log)
    assert [e[1] for e in log] == [k for k in KINDS if k in ("hsr", "text_anchored", "verify")]
