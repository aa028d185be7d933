"""Host logic of the fast attention kernel: its shared-memory plan.

The plan places a 64 KB table region at a shared address that is a multiple
of 65536 (the lookups merge a code byte into that address with one byte
permute), then as many stages of K codes, V codes and the two norm rows as
fit, in the space below and above the table. These tests check the plan's
invariants for every shape the kernel takes, on the numbers of a B200
(1 KB reserved before the dynamic region, 227 KB of it) and on others,
through the test hook `tq_test_attend_plan` (arithmetic only, no CUDA call).
"""

import itertools

import pytest

B200_RESERVED, B200_MAX_DYN = 1024, 232448
SHAPES = [(d, hw, nt, paged) for d, hw, nt, paged in itertools.product((128, 256), (4, 8, 16), (1, 2), (0, 1))
          if 16 % (hw * nt) == 0 and not (d == 256 and nt == 1 and hw == 4)]


@pytest.fixture(scope="module")
def plan_fn():
    from kv_cache_vector_turboquant_b200 import _binding

    return _binding.tq_test_attend_plan


def _regions(p):
    out = []
    for key, size in (("k", p["k_bytes"]), ("v", p["v_bytes"]), ("kn", p["norm_bytes"]), ("vn", p["norm_bytes"])):
        for s in range(8):
            off = p[key][s]
            if s < p["stages"]:
                assert off >= 0, (key, s)
                out.append((off, off + size, f"{key}{s}"))
            else:
                assert off == -1, (key, s)
    return out


def _check(p, reserved, max_dyn):
    assert p["stages"] % p["groups"] == 0 and p["stages"] >= 2 * p["groups"] and p["stages"] <= 8
    assert (reserved + p["table_off"]) % 65536 == 0
    assert p["table_off"] >= p["header_bytes"] and p["table_off"] + p["table_bytes"] <= max_dyn
    regs = _regions(p) + [(p["table_off"], p["table_off"] + p["table_bytes"], "table")]
    for lo, hi, name in regs:
        assert lo % 128 == 0 or name == "table", name
        assert p["header_bytes"] <= lo < hi <= max_dyn, name
    regs.sort()
    for (l0, h0, n0), (l1, h1, n1) in zip(regs, regs[1:]):
        assert h0 <= l1, (n0, n1)


# (d, nt) -> whether the launcher's kv-head counts per CTA (8 or 16 with one
# column tile, 4 or 8 with two) get a plan on a B200. At head_dim 256 with
# one column tile (at most 4 query heads per kv head) the stages of 8 or 16 kv
# heads do not fit beside the table, so those launches take the generic kernel.
EXPECT_PLAN = {(128, 1): True, (128, 2): True, (256, 1): False, (256, 2): True}


@pytest.mark.parametrize("d,hw,nt,paged", SHAPES)
def test_plan_on_b200_numbers(plan_fn, d, hw, nt, paged):
    st, p = plan_fn(d, hw, nt, paged, B200_RESERVED, B200_MAX_DYN)
    launcher_shape = hw in ((8, 16) if nt == 1 else (4, 8))
    if launcher_shape and not EXPECT_PLAN[d, nt]:
        assert st == 2
        return
    assert st == 0
    _check(p, B200_RESERVED, B200_MAX_DYN)
    assert p["groups"] == 16 // (hw * nt)
    assert p["k_bytes"] == 32 * hw * d // 2 and p["v_bytes"] == 32 * (hw * d // 4 + 16)
    assert p["header_bytes"] == 128 + (4 * 512 if paged else 0)


def test_benchmarked_step_plan(plan_fn):
    """d = 128, 8 kv heads per CTA, contiguous cache: the decode step's plan.
    A stage is 16,384 B of K codes, 8,704 of V codes (rows padded by 16 B)
    and two norm rows of 1,536 B (padded pitch); the 166,784 B around the
    table hold five such stages, and the stage count must be a multiple of
    the two warp groups: four."""
    st, p = plan_fn(128, 8, 1, 0, B200_RESERVED, B200_MAX_DYN)
    assert st == 0 and p["groups"] == 2 and p["table_off"] == 65536 - B200_RESERVED
    assert (p["k_bytes"], p["v_bytes"], p["norm_bytes"]) == (16384, 8704, 1536)
    assert B200_MAX_DYN - p["table_bytes"] - p["header_bytes"] == 166784
    assert p["stages"] == 4


@pytest.mark.parametrize("reserved", [0, 512, 1024, 4096, 65536 - 128, 65536])
def test_plan_for_other_reserved_offsets(plan_fn, reserved):
    """Wherever the dynamic region starts, the table lands on a 64 KB shared
    address past the header, or no plan is made."""
    for d, hw, nt, paged in SHAPES:
        st, p = plan_fn(d, hw, nt, paged, reserved, B200_MAX_DYN)
        if st == 0:
            _check(p, reserved, B200_MAX_DYN)
        else:
            assert st == 2


def test_plan_refuses_what_does_not_fit(plan_fn):
    assert plan_fn(128, 8, 1, 0, B200_RESERVED, 96 * 1024)[0] == 2  # no room for the table and two stages per group
    assert plan_fn(64, 8, 1, 0, B200_RESERVED, B200_MAX_DYN)[0] == 2  # head_dim 64 is not the fast kernel's
    assert plan_fn(256, 4, 1, 0, B200_RESERVED, B200_MAX_DYN)[0] == 2  # four groups of 2+ stages do not fit
    assert plan_fn(128, 8, 4, 0, B200_RESERVED, B200_MAX_DYN)[0] == 2  # 32 warps per tile
    assert plan_fn(128, 8, 1, 0, B200_RESERVED, 128 * 1024)[0] == 2  # table plus 4 stages need ~178 KB
    # a device with less shared memory: fewer stages (one warp group: any count from 2)
    st_full, p_full = plan_fn(128, 8, 2, 0, B200_RESERVED, B200_MAX_DYN)
    st, p = plan_fn(128, 8, 2, 0, B200_RESERVED, 200 * 1024)
    assert st_full == 0 and st == 0 and 2 <= p["stages"] < p_full["stages"]
    _check(p, B200_RESERVED, 200 * 1024)
