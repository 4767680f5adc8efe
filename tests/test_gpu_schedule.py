"""Scheduling of the tensor-core prefill: a resident CTA takes over the
tiles of CTAs that have not started, in the order given by a ticket counter
that a launch claims, counts on and frees, and launches take one of 64
counters in turn.  A tile is always computed by one CTA with the same instruction
sequence, so the output must not depend on which CTA computed which tile,
on the grid being smaller or larger than the SM count, on the launches
before it, or on other launches running at the same time on other streams:
every result here must be bitwise equal to a plain sequential run (whose
parity with the oracle the prefill tests establish).  A launch that finds
its counter held by another launch in flight must say so in its status word
(DA_ERR_SCHEDULE) rather than return an incomplete output with status 0."""
import random

import pytest
import torch

from differential_attention_sm_b200 import inputs as I
from parity import assert_status_ok, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from differential_attention_sm_b200 import binding
    binding.load()
    return binding


# (form, batch, seqlen, heads or (Hq, Hkv), causal, window): query-tile counts
# from 1 to well above the 148 SMs, ragged tails, both forms, windows
CASES = [
    ("v1", 1, 128, 1, True, 0),
    ("v1", 1, 200, 3, False, 0),
    ("v1", 2, 1000, 4, True, 0),
    ("v1", 2, 4096, 8, True, 0),
    ("v1", 1, 3000, 5, True, 700),
    ("v2", 1, 130, (2, 1), True, 0),
    ("v2", 2, 2048, (8, 2), True, 0),
    ("v2", 1, 5000, (16, 4), True, 1024),
    ("v2", 1, 777, (8, 4), False, 0),
]


def make_case(B, case, seed):
    form, b, n, h, causal, window = case
    dev = "cuda"
    if form == "v1":
        x = I.v1_inputs(b, n, h, 64, 128, seed)  # the tensor-core widths
        q, k, v = (x[t].to(dev) for t in ("q", "k", "v"))
        lam = torch.linspace(0.2, 0.9, h, device=dev)
        out = torch.empty(b, n, h, 128, dtype=torch.bfloat16, device=dev)

        def run(st, stream=None):
            if window:
                B.diffattn_v1_fwd_window(q, k, v, lam, window, causal=causal, apply_norm=True,
                                         lambda_init=0.3, out=out, dev_status=st,
                                         stream=stream)
            else:
                B.diffattn_v1_fwd(q, k, v, lam, causal=causal, apply_norm=True,
                                  lambda_init=0.3, out=out, dev_status=st, stream=stream)
            return out
    else:
        hq, hkv = h
        x = I.v2_inputs(b, n, hq, hkv, 128, seed)
        q, k, v, lam = (x[t].to(dev) for t in ("q", "k", "v", "lam"))
        out = torch.empty(b, n, hq // 2, 128, dtype=torch.bfloat16, device=dev)

        def run(st, stream=None):
            if window:
                B.diffattn_v2_prefill_window(q, k, v, lam, window, causal=causal, out=out,
                                             dev_status=st, stream=stream)
            else:
                B.diffattn_v2_prefill(q, k, v, lam, causal=causal, out=out, dev_status=st,
                                      stream=stream)
            return out
    return run, out


def reference_outputs(runs):
    refs = []
    for run in runs:
        st = status_word()
        refs.append(run(st).clone())
        torch.cuda.synchronize()
        assert_status_ok(st)
    return refs


def test_back_to_back_launches_of_every_size(B):
    runs = [make_case(B, c, 100 + i)[0] for i, c in enumerate(CASES)]
    refs = reference_outputs(runs)
    order = list(range(len(runs))) * 9  # 81 launches: every counter slot more than once
    random.Random(7).shuffle(order)
    st = status_word()
    for i in order:
        out = runs[i](st)
        assert torch.equal(out, refs[i]), f"case {CASES[i]} differs after reordering"
    torch.cuda.synchronize()
    assert_status_ok(st)


def test_concurrent_launches_on_several_streams(B):
    cases = [make_case(B, c, 200 + i) for i, c in enumerate(CASES)]
    runs = [run for run, _ in cases]
    refs = reference_outputs(runs)
    streams = [torch.cuda.Stream() for _ in runs]
    st = status_word()
    for rep in range(3):
        for _, out in cases:
            out.zero_()
        torch.cuda.synchronize()
        for run, s in zip(runs, streams):  # all in flight together
            with torch.cuda.stream(s):
                run(st, stream=s)
        torch.cuda.synchronize()
        for i, (_, out) in enumerate(cases):
            assert torch.equal(out, refs[i]), f"case {CASES[i]} differs (concurrent, rep {rep})"
    assert_status_ok(st)


def test_stopped_holder_is_taken_over(B):
    """A counter left held by a launch that stopped taking tickets (planted
    through the test hook; its word never changes) is taken over after about
    250 ms: the next launch is exact, with status 0."""
    run, _ = make_case(B, ("v1", 2, 1000, 4, True, 0), 300)
    ref = reference_outputs([run])[0]
    for slot in (0, 63):
        B.diffattn_selftest_hold_tile_counter(slot, 0x5EED0000 + slot, 3)
        st = status_word()
        out = run(st)
        torch.cuda.synchronize()
        assert_status_ok(st)
        assert torch.equal(out, ref)


def test_live_holder_beyond_the_wait_is_reported(B):
    """A counter kept held, as by a launch in flight, for longer than the 2 s
    bound: the waiting launch reports DA_ERR_SCHEDULE (it computes nothing,
    and says so); once the holder has freed it, the same launch is exact.
    diffattn_reset_tile_counters leaves every counter free."""
    run, _ = make_case(B, ("v2", 2, 2048, (8, 2), True, 0), 301)
    ref = reference_outputs([run])[0]
    keeper, waiter = torch.cuda.Stream(), torch.cuda.Stream()
    keeper.wait_stream(torch.cuda.current_stream())
    st = status_word()
    with torch.cuda.stream(keeper):
        B.diffattn_selftest_hold_tile_counter(20, 0xC0FFEE, 1, stream=keeper)
        held = torch.cuda.Event()
        held.record(keeper)
        B.diffattn_selftest_keep_tile_counter(20, 0xC0FFEE, 3000, stream=keeper)
    waiter.wait_event(held)
    with torch.cuda.stream(waiter):
        run(st, stream=waiter)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DA_ERR_SCHEDULE, B.status_string(int(st.item()))
    B.diffattn_reset_tile_counters()
    for _ in range(2):
        st = status_word()
        out = run(st)
        torch.cuda.synchronize()
        assert_status_ok(st)
        assert torch.equal(out, ref)


def test_overlapping_graph_replays_on_one_counter(B):
    """Two CUDA graphs captured onto the same counter (as two executions of
    one capture would be) and replayed at the same time on two streams: the
    later one waits for the earlier one's last ticket, so both are exact
    with status 0."""
    cases = [make_case(B, ("v1", 2, 4096, 8, True, 0), 310 + i) for i in range(2)]
    refs = reference_outputs([run for run, _ in cases])
    graphs, stats = [], []
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside capture
        for run, _ in cases:
            run(status_word())
    torch.cuda.synchronize()
    for run, _ in cases:
        st = status_word()
        g = torch.cuda.CUDAGraph()
        B.diffattn_selftest_hold_tile_counter(11, 0, 0)  # both captures take counter 11
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            run(st)
        graphs.append(g)
        stats.append(st)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for rep in range(20):
        for st, (_, out) in zip(stats, cases):
            st.zero_()
            out.zero_()
        for s_ in streams:
            s_.wait_stream(torch.cuda.current_stream())
        for g, s_ in zip(graphs, streams):
            with torch.cuda.stream(s_):
                g.replay()
        torch.cuda.synchronize()
        for i, (st, (_, out)) in enumerate(zip(stats, cases)):
            code = int(st.item())
            assert code == 0, "replay %d of graph %d: %s" % (rep, i, B.status_string(code))
            assert torch.equal(out, refs[i]), "replay %d of graph %d: wrong output" % (rep, i)
    del graphs
    torch.cuda.synchronize()
