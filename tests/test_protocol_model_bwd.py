"""The gradient kernels' barrier protocol (protocol_model_bwd) under random schedules: no race,
no parity aliasing, no deadlock, a clean exit after a timeout at any bounded wait, and the
planted protocol mistakes found."""
import itertools
import os
import re

import pytest

from protocol_model import ProtocolError
from protocol_model_bwd import BwdConfig, run_bwd

KINDS = ("dkdv", "dq")


@pytest.mark.parametrize("kind,stages,sets", list(itertools.product(KINDS, (3, 4), (2, 3))))
def test_bwd_protocol_holds_under_random_schedules(kind, stages, sets):
    for nit in range(0, 9):
        for seed in range(25):
            cfg = BwdConfig(kind=kind, nit=nit, stages=stages, sets=sets, tma_weight=(0.2 if seed % 3 == 0 else 1.0))
            run_bwd(cfg, seed * 131 + nit)


@pytest.mark.parametrize("kind,sets", list(itertools.product(KINDS, (2, 3))))
def test_bwd_timeout_at_any_wait_exits_cleanly(kind, sets):
    roles = ["tma", "mma"] + [f"grp{g}.{q}" for g in range(2) for q in range(4)]
    for nit in (1, 2, 5):
        for role in roles:
            for n in range(0, 5):
                for seed in range(3):
                    info = {}
                    run_bwd(BwdConfig(kind=kind, nit=nit, stages=4, sets=sets, timeout=(role, n)), seed * 7 + n, info)


PLANTS = [("empty_parity", "dkdv", 7, 2), ("prod_before_acc", "dkdv", 5, 2), ("prod_before_acc", "dq", 5, 3),
          ("no_s_full_wait", "dq", 4, 2), ("no_s_full_wait", "dkdv", 6, 3), ("lse_single_buffer", "dkdv", 6, 2),
          ("p_ready_per_group", "dkdv", 8, 3),
          ("p_ready_per_group", "dq", 8, 3), ("mma_skips_row_tmem", "dq", 4, 3),
          ("copy_without_row_full", "dq", 4, 3)]


SLOW = [(), ("grp1.0", "grp1.3"), ("grp0.2", "grp1.1"), ("mma",)]


@pytest.mark.parametrize("plant,kind,nit,sets", PLANTS)
def test_bwd_model_finds_planted_mistakes(plant, kind, nit, sets):
    with pytest.raises(ProtocolError):
        for seed in range(400):
            run_bwd(BwdConfig(kind=kind, nit=nit, stages=4, sets=sets, plant=plant,
                              tma_weight=0.3 if seed % 2 else 1.0, slow_roles=SLOW[seed % len(SLOW)]), seed)


def test_bwd_protocol_holds_with_late_warps():
    for kind, nit, seed, sets in itertools.product(KINDS, (1, 2, 3, 6), range(40), (2, 3)):
        run_bwd(BwdConfig(kind=kind, nit=nit, stages=4, sets=sets, slow_roles=SLOW[seed % len(SLOW)]), seed)


@pytest.mark.parametrize("plant", ["no_tma_drain", "no_mma_drain"])
def test_bwd_model_finds_a_missing_drain(plant):
    roles = ["tma", "mma"] + [f"grp{g}.{q}" for g in range(2) for q in range(4)]
    with pytest.raises(ProtocolError, match="in flight"):
        for role, n, seed in itertools.product(roles, range(4), range(6)):
            run_bwd(BwdConfig(kind="dkdv", nit=5, stages=3, plant=plant, timeout=(role, n), tma_weight=0.05), seed)


def test_bwd_model_barriers_match_the_kernel_source():
    """The arrival counts and the group barrier width the model assumes are the kernel's."""
    src = open(os.path.join(os.path.dirname(__file__), "..", "exact_attention_sdpa_b200", "csrc",
                            "attn_bwd_tc.cuh")).read()
    inits = dict(re.findall(r"mbar_init\(&br\.(\w+)(?:\[\w+\])?, (\d+)\)", src))
    assert inits == {"row_full": "1", "row_tmem": "256", "full": "1", "empty": "1", "s_full": "1", "p_ready": "128",
                     "acc_done": "1"}
    assert "bar.red.and.pred q, %2, 128, p;" in src
    assert re.search(r"constexpr int kMmaWarp = 8, kTmaWarp = 9;", src)
    # column sets: 3 for dQ and, where tensor memory holds them beside dK and dV, for dK/dV
    assert "static constexpr int kSets = (3 * 128 + 2 * D <= 512 && kStages >= 5) ? 3 : 2;" in src
    assert "static constexpr int kSets = (kStages >= 5) ? 3 : 2;" in src
    assert "        sm100::mbar_init(&br.s_full[c], 1);\n        sm100::mbar_init(&br.p_ready[c], 128);" in src


def test_dq_d_read_guard_is_a_second_guard():
    """A dQ group without a block reading D would race group 0's store over chunk 0 -- but every
    group arrives on row_tmem (after its D read) before the first product can run, so that
    arrival orders the read as well; the kernel's `nit > g` guard is kept as a second one."""
    for seed in range(300):
        run_bwd(BwdConfig(kind="dq", nit=1, stages=4, sets=3, plant="dq_reads_d_without_block",
                          slow_roles=SLOW[seed % len(SLOW)]), seed)
