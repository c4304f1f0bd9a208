"""The one-launch tail's host planner, without a device (moe_debug_tail_plan).

The planner places in a CTA's shared memory the raw stages (one unit's two
128-row tiles of one 256-wide K chunk of the pack's tiled planes, for the
larger of the two projections' formats), the B slots (the group's slot rows,
16-row TMA boxes of 128 bytes) and, overlaid on them, the routing and planning
scratch; the A stages live in tensor memory.  These checks hold the layout the
kernel relies on: alignments of the TMA and bulk-copy destinations, the ring
depths its barriers are sized for, and the shared-memory budget."""
import pytest

import block_quantized_expert_moe_b200 as bq

SMEM_MAX = 225 * 1024  # dynamic shared memory the planner may use per CTA
GRID = 148             # B200 SMs

# bytes of one tiled block (128 rows x 256 of K) per format: codes, scales, Q5_1 fifth bits
TILE = {bq.MOE_FMT_Q8_0: 128 * 256 + 128 * 16, bq.MOE_FMT_Q5_1: 128 * 128 + 128 * 32 + 128 * 32,
        bq.MOE_FMT_IQ4_NL: 128 * 128 + 128 * 16, bq.MOE_FMT_NVFP4: 128 * 128 + 128 * 16}
DEVICE_FMT = {bq.MOE_FMT_Q5_0: bq.MOE_FMT_Q5_1}

PAIRS = [(bq.MOE_FMT_IQ4_NL, bq.MOE_FMT_Q5_1), (bq.MOE_FMT_NVFP4, bq.MOE_FMT_NVFP4),
         (bq.MOE_FMT_Q8_0, bq.MOE_FMT_Q8_0), (bq.MOE_FMT_Q5_0, bq.MOE_FMT_IQ4_NL), (bq.MOE_FMT_Q5_1, bq.MOE_FMT_Q8_0)]


def _plan(T, max_tokens, H=2048, E=512, I=512, k=10, dt=bq.MOE_DT_BF16, fg=bq.MOE_FMT_IQ4_NL,
          fd=bq.MOE_FMT_Q5_1, grid=GRID):
    return bq.moe_debug_tail_plan(T, max_tokens, H, E, I, k, dt, fg, fd, grid)


@pytest.mark.parametrize("fg,fd", PAIRS)
@pytest.mark.parametrize("T,max_tokens", [(1, 8), (2, 8), (8, 8), (13, 16), (33, 64), (64, 64)])
@pytest.mark.parametrize("dt", [bq.MOE_DT_BF16, bq.MOE_DT_F32])
def test_model_shapes_fit_with_aligned_rings(fg, fd, T, max_tokens, dt):
    p = _plan(T, max_tokens, dt=dt, fg=fg, fd=fd)
    assert p["fits"], p
    raw = 2 * max(TILE[DEVICE_FMT.get(fg, fg)], TILE[DEVICE_FMT.get(fd, fd)])
    assert p["raw_stage_bytes"] == raw
    assert p["b_slot_bytes"] == ((min(max_tokens, 64) + 15) // 16 * 16) * 128
    # 128-byte-swizzled TMA / MMA operands need 1024-byte alignment: every raw stage and
    # B slot starts at a multiple of 1024 from the 1024-aligned base
    assert p["raw_stage_bytes"] % 1024 == 0 and p["b_slot_bytes"] % 2048 == 0
    assert 2 <= p["raw_stages"] <= 4 and 4 <= p["b_slots"] <= 8 and p["a_stages"] == 4
    rings = p["raw_stages"] * p["raw_stage_bytes"] + p["b_slots"] * p["b_slot_bytes"]
    assert p["rings_bytes"] >= rings
    assert p["rings_bytes"] < p["smem_bytes"] <= SMEM_MAX


def test_deeper_rings_when_shared_memory_allows():
    small = _plan(8, 8)                    # 16-row B slots
    large = _plan(64, 64)                  # 64-row B slots take more of the budget
    assert small["raw_stages"] >= large["raw_stages"]
    assert small["raw_stages"] * small["raw_stage_bytes"] + small["b_slots"] * small["b_slot_bytes"] <= SMEM_MAX


@pytest.mark.parametrize("kw", [dict(T=65, max_tokens=65), dict(T=8, max_tokens=4), dict(T=8, max_tokens=8, k=17),
                                dict(T=8, max_tokens=8, H=2048 + 128), dict(T=8, max_tokens=8, I=512 + 64),
                                dict(T=8, max_tokens=8, E=1025), dict(T=0, max_tokens=8)])
def test_shapes_the_tail_does_not_take(kw):
    T, mt = kw.pop("T"), kw.pop("max_tokens")
    p = _plan(T, mt, **kw)
    assert not p["fits"] and p["smem_bytes"] == 0


def test_small_layer_and_argument_checks():
    # the smoke layer's shape: H 1024, 64 experts, I 256, top-8, fp32 tokens, Q8_0
    p = _plan(4, 4, H=1024, E=64, I=256, k=8, dt=bq.MOE_DT_F32, fg=bq.MOE_FMT_Q8_0, fd=bq.MOE_FMT_Q8_0)
    assert p["fits"] and p["smem_bytes"] <= SMEM_MAX
    with pytest.raises(bq.MoeError):
        bq.moe_debug_tail_plan(8, 8, 2048, 512, 512, 10, bq.MOE_DT_BF16, 9, bq.MOE_FMT_Q5_1, GRID)
    with pytest.raises(bq.MoeError):
        bq.moe_debug_tail_plan(8, 8, 2048, 512, 512, 10, 7, bq.MOE_FMT_IQ4_NL, bq.MOE_FMT_Q5_1, GRID)
