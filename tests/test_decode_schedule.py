"""The decode driver's host-side schedule (query_aware_sparse_tb_b200.decode)
against the oracle's independently written schedule (oracle.schedule), on CPU:
projection batches, prediction steps, producer layers and query slots."""
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
