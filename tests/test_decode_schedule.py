"""The decode driver's host-side schedule (query_aware_sparse_tb_b200.decode)
against the oracle's independently written schedule (oracle.schedule), on CPU:
projection batches, prediction steps, producer layers and query slots; and the
driver's own launch order: which attention launches may prefetch, and how a
prediction step's selections are spread over streams (faked on the host)."""
from oracle import schedule as oschedule
from query_aware_sparse_tb_b200 import decode


def test_projection_schedule_matches_oracle_schedule():
    for ctx0 in ([299], [700, 641, 5000], [64, 128], [1, 63, 65]):
        for N in (1, 16, 64):
            pre, ev = decode.projection_schedule(ctx0, N, 200)
            for b, t0 in enumerate(ctx0):
                opre, oev = oschedule.projection_events(t0, N, 200)
                assert pre[b] == opre
                assert [(i, v[b]) for i, v in sorted(ev.items()) if v[b] >= 0] == oev
            # an event lists every sequence; one that projects nothing there gets -1
            assert all(len(v) == len(ctx0) and any(x >= 0 for x in v) for v in ev.values())


def test_prediction_steps_match_oracle_schedule():
    for P in (1, 4, 16):
        assert [i for i in range(100) if decode.is_prediction_step(i, P)] == \
            [i for i in range(100) if oschedule.is_prediction_step(i, P)]


def test_producers_and_slots_match_oracle_schedule():
    for stride in (1, 2, 4):
        for layer in range(32):
            assert decode.producer_layer(layer, stride) == oschedule.producer_of(layer, stride)
            assert decode.query_slot(layer, stride) == oschedule.slot_of(layer, stride)
            assert decode.producer_layer(layer, stride) + decode.query_slot(layer, stride) == layer


def test_attention_prefetch_only_where_the_contract_holds():
    # the decoder asks for TB_ATTN_PREFETCH_KV on every attention launch except
    # the first one right after the selection of the same (only) layer, whose
    # selection words the preceding kernel has just written
    from query_aware_sparse_tb_b200 import _lib as L

    class Rec(decode.SparseDecoder):
        def __init__(self, n_layers, interval, prefetch_kv):
            self.shape = decode.DecodeShape(batch=1, n_layers=n_layers, n_q_heads=8, n_kv_heads=2, head_dim=64,
                                            d_proj=16, hidden=0, inter=0, stride=1, sink=4, window=16, budget=8,
                                            nbr=1, interval=interval, ctx_cap=512)
            self.prefetch_kv = prefetch_kv
            self.overlap_select = False  # (one stream: no GPU here)
            self.proj_begin, self.qp, self.calls = {}, {}, []

        def select(self, step, layer, qp_direct=None, stream=None, ws_sel=None, ws_plan=None):
            self.calls.append(("select", step, layer))

        def attend(self, step, layer, Q, out, stream=None, prefetch=False):
            self.calls.append(("attend", step, layer, prefetch))

    for n_layers in (1, 3):
        for interval in (1, 4):
            for prefetch_kv in (False, True):
                dec = Rec(n_layers, interval, prefetch_kv)
                for i in range(6):
                    dec.step(i, [None] * n_layers, [None] * n_layers, qp_direct=[None] * n_layers)
                modes = [(c[1], c[2], c[3]) for c in dec.calls if c[0] == "attend"]
                assert len(modes) == 6 * n_layers
                for step, layer, pf in modes:
                    right_after_own_select = n_layers == 1 and step % interval == 0
                    assert pf == (prefetch_kv and not right_after_own_select), (n_layers, interval, step, layer)
    assert L.TB_ATTN_WAIT_ALL == 0 and L.TB_ATTN_PREFETCH_KV == 1


def test_last_selection_on_the_callers_stream():
    # with the selections round-robin over n streams, the caller's stream
    # issues layers 0, n, 2n, ...; the first attention launch after them may
    # prefetch only when the last of those is not layer 0
    f = decode.main_stream_last_selected
    assert [f(1, 1), f(3, 1), f(32, 1)] == [0, 2, 31]
    assert [f(4, 4), f(5, 4), f(32, 4), f(4, 2), f(2, 4), f(32, 2)] == [0, 4, 28, 2, 0, 30]


def test_selection_streams_fork_route_and_join(monkeypatch):
    # a prediction step with the selections spread over n streams, with the
    # streams and events faked on the host: every extra stream (and the
    # predictors' stream) waits for an event recorded on the caller's stream
    # first; the producers' predictor calls run on their own stream with an
    # event after each; layer l's selection goes to stream l mod n with that
    # stream's own workspaces, after a wait for its producer's event; the
    # caller's stream waits for the predictors' last event and for an event
    # recorded on every extra stream after its last selection, before the
    # first attention launch
    import torch
    log = []

    class FakeStream:
        def __init__(self, name):
            self.name = name

        def wait_event(self, ev):
            log.append(("wait", self.name, ev.id))

    class FakeEvent:
        n = 0

        def __init__(self):
            FakeEvent.n += 1
            self.id = FakeEvent.n

        def record(self, stream):
            log.append(("record", stream.name, self.id))

    main = FakeStream("main")
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: main)

    class Rec(decode.SparseDecoder):
        def __init__(self, n_layers, n_streams):
            self.shape = decode.DecodeShape(batch=1, n_layers=n_layers, n_q_heads=8, n_kv_heads=2, head_dim=64,
                                            d_proj=16, hidden=16, inter=16, stride=4, sink=4, window=16, budget=8,
                                            nbr=1, interval=4, ctx_cap=512)
            self.device = "cuda"
            self.prefetch_kv = True
            self.overlap_select = n_streams > 1
            self.sel_lanes = [(FakeStream(f"lane{k}"), f"ws_sel{k}", f"ws_plan{k}") for k in range(1, n_streams)]
            self.pred_stream = FakeStream("pred") if n_streams > 1 else None
            self.producers = [l for l in range(n_layers) if l % 4 == 0]
            self.proj_begin, self.qp = {}, {p: None for p in self.producers}

        def predict(self, producer, h, stream=None):
            log.append(("predict", producer, getattr(stream, "name", "main")))

        def select(self, step, layer, qp_direct=None, stream=None, ws_sel=None, ws_plan=None):
            log.append(("select", layer, getattr(stream, "name", "main"), ws_sel, ws_plan))

        def attend(self, step, layer, Q, out, stream=None, prefetch=False):
            log.append(("attend", layer, prefetch))

    for n_layers, n_streams in ((8, 4), (6, 4), (4, 4), (5, 2), (3, 1)):
        log.clear()
        dec = Rec(n_layers, n_streams)
        dec.step(0, [None] * n_layers, [None] * n_layers, h=[None] * len(dec.producers))
        spread = n_streams > 1
        kinds = [e[0] for e in log]
        first_select = kinds.index("select")
        preds = [e for e in log[:first_select] if e[0] == "predict"]
        assert [e[1] for e in preds] == dec.producers
        assert all(e[2] == ("pred" if spread else "main") for e in preds)
        sels = [e for e in log if e[0] == "select"]
        assert [e[1] for e in sels] == list(range(n_layers))
        for _, l, st, ws, wp in sels:
            k = l % n_streams
            assert st == ("main" if k == 0 else f"lane{k}")
            assert (ws, wp) == ((None, None) if k == 0 else (f"ws_sel{k}", f"ws_plan{k}"))
        if not spread:
            assert "record" not in kinds and "wait" not in kinds
        else:
            # the fork: one event on the caller's stream, before anything else
            assert log[0][:2] == ("record", "main")
            fork = log[0][2]
            forked = sorted(e[1] for e in log[:first_select] if e[0] == "wait" and e[2] == fork)
            assert forked == sorted([f"lane{k}" for k in range(1, n_streams)] + ["pred"])
            # an event on the predictors' stream after each predictor call
            ready = {}
            for i, e in enumerate(log):
                if e[0] == "predict":
                    assert log[i + 1][:2] == ("record", "pred")
                    ready[e[1]] = log[i + 1][2]
            # each selection right after its stream waits for its producer's event
            for i, e in enumerate(log):
                if e[0] == "select":
                    assert log[i - 1] == ("wait", e[2], ready[decode.producer_layer(e[1], 4)])
            # the join: the caller's stream waits for the predictors and every extra stream
            first_attend = kinds.index("attend")
            tail = log[max(i for i, e in enumerate(log) if e[0] == "select") + 1:first_attend]
            joins = {e[1]: e[2] for e in tail if e[0] == "record"}
            assert sorted(joins) == [f"lane{k}" for k in range(1, n_streams)]
            waited = sorted(e[2] for e in tail if e[0] == "wait" and e[1] == "main")
            assert waited == sorted(list(joins.values()) + [ready[max(ready)]])
        attends = [e for e in log if e[0] == "attend"]
        assert [e[1] for e in attends] == list(range(n_layers))
        # the first launch may prefetch unless the caller's stream selected layer 0 last
        assert attends[0][2] == (decode.main_stream_last_selected(n_layers, n_streams) != 0)
        assert all(e[2] for e in attends[1:])
