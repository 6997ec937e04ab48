"""Host logic of the staggered window schedule (no GPU): every sequence steps through its window
once per cycle, exactly one window end per sequence per cycle, and the phases spread the window
ends evenly over the steps."""

import torch

from recurrent_state_read_b200.decode import stagger_plan


def test_stagger_plan_cycles_every_sequence_through_its_window():
    B, W = 13, 4
    plan = stagger_plan(B, W, "cpu")
    assert len(plan) == W
    js = torch.stack([jv for jv, _ in plan])  # [W, B]
    for b in range(B):
        seq = js[:, b].tolist()
        assert sorted(seq) == [0] + list(range(1, W))  # steps 1..W-1 from the sketch, one window end
        end = seq.index(0)
        for s in range(1, W):  # consecutive steps advance by one, wrapping after the window end
            assert seq[(end + s) % W] == s
    for s, (jv, seqs) in enumerate(plan):
        assert seqs.dtype == torch.int32 and jv.dtype == torch.int32
        assert sorted(seqs.tolist()) == [b for b in range(B) if jv[b] == 0]
        assert abs(len(seqs) - B / W) < 1  # window ends spread evenly


def test_stagger_plan_window_one():
    plan = stagger_plan(5, 1, "cpu")
    (jv, seqs), = plan
    assert jv.tolist() == [0] * 5 and seqs.tolist() == list(range(5))  # every step is a window end
