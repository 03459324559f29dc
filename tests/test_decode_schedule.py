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
