"""Host-side order of the wave-scheduled expert-parallel step (DeepSeek V4
infra notes, §6.1 "MegaMoE": the experts go in waves, the rows of wave w + 1
travelling while wave w computes).

EPMoELayer.forward(..., waves=n) and VirtualEP.forward(..., waves=n) are run
on the CPU with recording stand-ins for the C-ABI phases, the peer barrier,
CUDA streams and events, and the recorded order is checked:

* every rank issues its barriers with strictly rising epochs in one fixed
  order (route, the n sends, the results), whatever n is, so ranks that pass
  the same n meet at the same barriers;
* wave w's expert GEMMs run on the compute stream only after an event
  recorded behind wave w's send (and, across processes, its barrier) on the
  communication stream, and waves keep their order on each stream;
* the combine runs on the caller's stream after it has waited for both.
"""
import types

import pytest
import torch

import deterministic_expert_b200 as moe


class _Log:
    def __init__(self):
        self.ops = []

    def add(self, *op):
        self.ops.append(op)


class _Stream:
    def __init__(self, log, name):
        self.log, self.name, self.cuda_stream = log, name, 0

    def wait_event(self, ev):
        self.log.add(self.name, "wait", ev.id)

    def wait_stream(self, other):
        self.log.add(self.name, "wait_stream", other.name)


def _install_fakes(monkeypatch, log, names):
    counter = {"event": 0}

    class _Event:
        def __init__(self, *a, **k):
            counter["event"] += 1
            self.id = counter["event"]

        def record(self, stream):
            log.add(stream.name, "record", self.id)

    it = iter(names)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "Stream", lambda *a, **k: _Stream(log, next(it)))
    monkeypatch.setattr(moe, "peer_barrier",
                        lambda flags, rank, epoch, err, limit, stream: log.add(stream.name, "barrier", epoch))


class _Rank:
    def __init__(self, log, E, k, tag=""):
        self.log, self.tag = log, tag
        self.cfg = types.SimpleNamespace(E=E, k=k)

    def route(self, x, ids, xbuf, stream=None):
        self.log.add(_name(stream), "route" + self.tag)

    def send(self, T, peers, stream=None, wave=None, n_waves=1):
        self.log.add(_name(stream), "send" + self.tag, wave)

    def experts(self, T, peers, stream=None, wave=None, n_waves=1):
        self.log.add(_name(stream), "experts" + self.tag, wave)

    def combine(self, residual, xbuf, on, orr, idx=None, w=None, stream=None):
        self.log.add(_name(stream), "combine" + self.tag)


def _name(stream):
    return stream.name if stream is not None else "main"


def _ep_layer(log, world=2, rank=0, E=8, k=2):
    layer = object.__new__(moe.EPMoELayer)
    layer.world, layer.rank = world, rank
    layer.me = _Rank(log, E, k)
    layer.peers = types.SimpleNamespace(xbuf=[0] * world)
    layer._flags = [0] * world
    layer.err = torch.zeros(1, dtype=torch.int32)
    layer.limit_us = 1000
    layer._epoch = 0
    layer._comm = layer._comp = None
    return layer


@pytest.mark.parametrize("waves", [1, 2, 4])
def test_ep_layer_wave_order(monkeypatch, waves):
    log = _Log()
    _install_fakes(monkeypatch, log, ["comm", "comp"])
    layer = _ep_layer(log)
    main = _Stream(log, "main")
    x = torch.zeros((5, 16), dtype=torch.bfloat16)
    for step in range(2):
        log.ops.clear()
        layer.forward(x, x.clone(), stream=main, waves=waves)
        ops = log.ops
        barriers = [op for op in ops if op[1] == "barrier"]
        epochs = [op[2] for op in barriers]
        # route, one per wave's send, the results: strictly rising, continuing across steps
        assert len(barriers) == waves + 2
        assert epochs == list(range(step * (waves + 2) + 1, (step + 1) * (waves + 2) + 1))
        assert ops[0] == ("main", "route") and ops[1][0:2] == ("main", "barrier")
        assert ops[-1] == ("main", "combine")
        if waves == 1:
            assert [op[1] for op in ops] == ["route", "barrier", "send", "barrier", "experts", "barrier", "combine"]
            assert all(op[0] == "main" for op in ops)
            continue
        pos = {op: i for i, op in enumerate(ops)}
        for w in range(waves):
            send = ops.index(("comm", "send", w))
            bar = next(i for i in range(send, len(ops)) if ops[i][0:2] == ("comm", "barrier"))
            rec = next(i for i in range(bar, len(ops)) if ops[i][0:2] == ("comm", "record"))
            wait = ops.index(("comp", "wait", ops[rec][2]))
            exp = ops.index(("comp", "experts", w))
            assert send < bar < rec < wait < exp, w
            if w:
                assert ops.index(("comm", "send", w - 1)) < send
                assert ops.index(("comp", "experts", w - 1)) < exp
        # the results barrier follows the last wave's GEMMs on the compute stream,
        # and the combine follows both joins
        last = ops.index(("comp", "experts", waves - 1))
        final = [i for i, op in enumerate(ops) if op[0:2] == ("comp", "barrier")]
        assert len(final) == 1 and final[0] > last
        comb = ops.index(("main", "combine"))
        assert ops.index(("main", "wait_stream", "comm")) < comb
        assert ops.index(("main", "wait_stream", "comp")) < comb
        assert len(pos) == len(ops)


def test_ep_layer_rejects_bad_wave_counts(monkeypatch):
    log = _Log()
    _install_fakes(monkeypatch, log, ["comm", "comp"])
    layer = _ep_layer(log, E=8, world=2)          # 4 experts per rank
    x = torch.zeros((3, 16), dtype=torch.bfloat16)
    for waves in (0, 5):
        with pytest.raises(ValueError):
            layer.forward(x, x.clone(), waves=waves)
    assert log.ops == []                          # nothing was issued


@pytest.mark.parametrize("world,waves", [(2, 2), (4, 2), (2, 4)])
def test_virtual_ep_wave_order(monkeypatch, world, waves):
    log = _Log()
    _install_fakes(monkeypatch, log, ["comm", "comp"])
    ep = object.__new__(moe.VirtualEP)
    ep.world, ep.E_loc = world, 8 // world
    ep.ranks = [_Rank(log, 8, 2, tag=str(r)) for r in range(world)]
    ep.xbuf = [torch.zeros(256, dtype=torch.uint8) for _ in range(world)]
    ep.peers = types.SimpleNamespace(xbuf=[0] * world)
    ep._comm, ep._comp = _Stream(log, "comm"), _Stream(log, "comp")
    main = _Stream(log, "main")
    xs = [torch.zeros((3, 16), dtype=torch.bfloat16) for _ in range(world)]
    ep.forward(xs, [x.clone() for x in xs], stream=main, waves=waves)
    ops = log.ops
    # every rank routes before anything else, and combines last, on the caller's stream
    assert [op for op in ops[:world]] == [("main", f"route{r}") for r in range(world)]
    assert [op for op in ops[-world:]] == [("main", f"combine{r}") for r in range(world)]
    for w in range(waves):
        sends = [ops.index(("comm", f"send{r}", w)) for r in range(world)]
        exps = [ops.index(("comp", f"experts{r}", w)) for r in range(world)]
        rec = next(i for i in range(max(sends), len(ops)) if ops[i][0:2] == ("comm", "record"))
        wait = ops.index(("comp", "wait", ops[rec][2]))
        # every rank's send of wave w, then the event, then every rank's GEMMs of wave w
        assert max(sends) < rec < wait < min(exps), w
    assert ops.index(("main", "wait_stream", "comm")) < len(ops) - world
    assert ops.index(("main", "wait_stream", "comp")) < len(ops) - world
