"""The fused layer body's work list (bpt_layer_tail_plan), on the host.

"Blockwise Parallel Transformer — BPT", section "The fused blockwise
algorithm": the body after attention (y, LN2, the FFN) runs once for every
query block.  The layer body deals items of two query blocks round-robin over
its CTA pairs and shares the items of a last round that would keep at most
half of the pairs busy: two pairs each compute half of such an item's
columns.  The plan comes from the code the kernel runs (compiled for the host
too), so these checks need no GPU; the GPU tests show the same counts in the
hand-over counters and the output bitwise equal to the waves schedule.
"""
import pytest

import blockwise_attn_ffn_b200 as bpt


def covered(B, N, d, h, d_ff, resident):
    st, P, L, plan = bpt.bpt_layer_tail_plan(B, N, d, h, d_ff, True, resident)
    assert st == bpt.BPT_OK
    items = (B * ((N + 127) // 128) + 1) // 2
    assert P == min(resident, items) and len(plan) == P
    whole, halves = {}, {}
    for q, (J, Jfull, hitem, half, partner) in enumerate(plan):
        for j in range(Jfull):
            it = q + j * P
            assert it not in whole
            whole[it] = q
        if half >= 0:
            assert J == Jfull + 1 and half in (0, 1) and 0 <= partner < P and partner != q
            assert hitem not in whole
            halves.setdefault(hitem, {})[half] = (q, partner)
        else:
            assert (J, hitem, partner) == (Jfull, -1, -1)
    # every item once: whole, or as the two halves of two partner pairs
    assert sorted(list(whole) + list(halves)) == list(range(items))
    for it, hv in halves.items():
        assert set(hv) == {0, 1}, it
        (q0, p0), (q1, p1) = hv[0], hv[1]
        assert p0 == q1 and p1 == q0
    assert len(halves) == L
    span = max(Jfull + (0.5 if half >= 0 else 0.0) for _, Jfull, _, half, _ in plan)
    return P, L, items, span


@pytest.mark.parametrize("B,N,d,h,d_ff,resident,want_P,want_L,want_span", [
    # long-context layer: 256 items on 74 pairs, 34 shared, 3.5 items per pair at most
    (1, 65536, 2048, 16, 8192, 74, 74, 34, 3.5),
    # fewer resident pairs: 256 = 4 x 60 + 16, shared; 256 = 3 x 72 + 40 > 36, whole
    (1, 65536, 2048, 16, 8192, 60, 60, 16, 4.5),
    (1, 65536, 2048, 16, 8192, 72, 72, 0, 4.0),
    # ragged sequence: 168 blocks = 84 items, 10 shared
    (1, 128 * 167 + 78, 1024, 8, 1024, 74, 74, 10, 1.5),
    # the most shared items (37 = 74 / 2) and one past it (38: whole)
    (6, 128 * 37 - 5, 1024, 16, 1536, 74, 74, 37, 1.5),
    (1, 128 * 224, 1024, 8, 1024, 74, 74, 0, 2.0),
    # halves need d % 1024 == 0 and d_ff % 512 == 0
    (1, 128 * 168, 1536, 12, 1024, 74, 74, 0, 2.0),
    (1, 128 * 168, 1024, 8, 1792, 74, 74, 0, 2.0),
    # no item left over, fewer items than pairs, one odd block
    (1, 128 * 148, 1024, 8, 1024, 74, 74, 0, 1.0),
    (1, 16384, 1024, 16, 4096, 74, 64, 0, 1.0),
    (1, 128 * 149, 1024, 8, 1536, 74, 74, 1, 1.5),
])
def test_every_item_runs_once(B, N, d, h, d_ff, resident, want_P, want_L, want_span):
    P, L, items, span = covered(B, N, d, h, d_ff, resident)
    assert (P, L, span) == (want_P, want_L, want_span), (P, L, items, span)


def test_plan_rows_and_empty_layer():
    st, P, L, plan = bpt.bpt_layer_tail_plan(1, 65536, 2048, 16, 8192, True, 74, rows=3)
    assert st == bpt.BPT_OK and (P, L, len(plan)) == (74, 34, 3)
    st, P, L, plan = bpt.bpt_layer_tail_plan(1, 65536, 2048, 16, 8192, True, 74, rows=0)
    assert st == bpt.BPT_OK and (P, L, plan) == (74, 34, [])
    st, P, L, plan = bpt.bpt_layer_tail_plan(0, 1024, 1024, 8, 1024, True, 74)
    assert st == bpt.BPT_OK and (P, L, plan) == (0, 0, [])


@pytest.mark.parametrize("args,expect", [
    ((1, 4096, 1024, 8, 1024, True, 0), bpt.BPT_ERR_INVALID_ARG),
    ((1, 4096, 1024, 8, 1024, True, bpt.BPT_TAIL_MAX_PAIRS + 1), bpt.BPT_ERR_INVALID_ARG),
    ((1, 4096, 1024, 3, 1024, True, 74), bpt.BPT_ERR_INVALID_ARG),   # d % h != 0
    ((1, 4096, 1024, 4, 1024, True, 74), bpt.BPT_ERR_UNSUPPORTED),   # d_k = 256
])
def test_rejects_bad_arguments(args, expect):
    assert bpt.bpt_layer_tail_plan(*args)[0] == expect
