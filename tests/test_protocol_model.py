"""The forward kernel's mbarrier protocol, executed as a model under random schedules (CPU).

tests/protocol_model.py restates the barrier protocol of attn_fwd_kernel.cuh: one actor per
warp, asynchronous tensor-core and TMA work, version-tagged buffers, and the abort path of the
bounded waits.  These tests run it over the kernel's configurations (separate P columns at
d <= 64 or P inside S at d = 128, causal or not, K/V ring depths 2-4, staged bias tiles) and
over random unit sequences, including units of a single key tile and causal units whose second
query tile reaches one more key tile than the first.  Every run must finish without a stale
read, a parity-aliased wait or a deadlock.  With a timeout forced at any wait of any role,
every role must still reach the teardown, with no TMA load or tensor-core operation in flight
when tensor memory is freed.  Other tests plant protocol mistakes of the kinds a change to the
kernel could make and check that the model finds each of them.
"""
import random

import pytest

import protocol_model as pm

CONFIGS = [
    # (separate_p, causal, stages, bias_stages): the kernel's instantiations at d = 32, 64, 128
    (True, True, 4, 0), (True, True, 4, 2), (True, False, 4, 2),     # d = 32 (bias: 2 stages)
    (True, True, 3, 0), (True, False, 3, 0), (True, True, 3, 1), (True, False, 3, 1),   # d = 64
    (False, True, 2, 0), (False, False, 2, 0),                        # d = 128
    (True, True, 2, 0), (False, True, 3, 0),                          # other ring depths
]


@pytest.mark.parametrize("sep,causal,stages,bias", CONFIGS)
def test_protocol_holds_under_random_schedules(sep, causal, stages, bias):
    for rep in range(40):
        rng = random.Random(1000 * stages + 10 * bias + rep)
        cfg = pm.Config(separate_p=sep, causal=causal, stages=stages, bias_stages=bias,
                        units=pm.random_units(rng, causal, rng.randint(1, 4)),
                        tma_weight=0.03 if rep % 4 >= 2 else 1.0)
        pm.run(cfg, seed=rep)


@pytest.mark.parametrize("sep", [True, False])
def test_protocol_holds_over_long_unit_sequences(sep):
    # many units per CTA: every parity counter wraps many times
    for rep in range(6):
        rng = random.Random(77 + rep)
        cfg = pm.Config(separate_p=sep, causal=True, stages=3 if sep else 2,
                        units=pm.random_units(rng, True, 12, max_tiles=3))
        pm.run(cfg, seed=rep)


def test_single_tile_units_back_to_back():
    # units with one key tile each: S_i(0) of the next unit, Q release and the statistics
    # double buffer are exercised on every unit
    for rep in range(20):
        cfg = pm.Config(separate_p=rep % 2 == 0, causal=True, stages=3,
                        units=[(1, 1 + (rep + u) % 2) for u in range(6)])
        pm.run(cfg, seed=rep)


ROLES = ["tma", "mma", "mma0", "mma1"] + [f"softmax{i}.{q}" for i in range(2) for q in range(4)] + \
    [f"epi.{q}" for q in range(4)]


@pytest.mark.parametrize("sep,causal,stages,bias", [(True, True, 3, 0), (True, False, 4, 2), (True, True, 3, 1),
                                                    (False, True, 2, 0), (False, False, 2, 0)])
def test_a_timeout_at_any_wait_drains_and_exits(sep, causal, stages, bias):
    # every role, every one of its first bounded waits: the wait gives up (as after the kernel's
    # clock64 limit), the abort flag goes up, and every role must still leave its loops, the
    # producer and the MMA warp must drain, and nothing may be in flight at teardown
    units = [(2, 3), (1, 1), (3, 3)] if causal else [(2, 2), (1, 1), (3, 3)]
    aborted = 0
    for role in ROLES:
        for idx in range(10):
            info = {}
            cfg = pm.Config(separate_p=sep, causal=causal, stages=stages, bias_stages=bias, units=units,
                            timeout=(role, idx))
            pm.run(cfg, seed=idx, info=info)
            aborted += info["aborted"]
    assert aborted >= 100, aborted


@pytest.mark.parametrize("plant", ["no_tma_drain", "no_mma_drain"])
def test_model_finds_a_missing_drain(plant):
    for rep in range(200):
        rng = random.Random(rep)
        causal = rep % 4 != 0         # every other d <= 64 run non-causal: the two tile issuers
        cfg = pm.Config(separate_p=rep % 2 == 0, causal=causal, stages=3 if rep % 2 == 0 else 2,
                        units=pm.random_units(rng, causal, 2, max_tiles=3), plant=plant,
                        timeout=(rng.choice(ROLES), rng.randint(0, 4)))
        try:
            pm.run(cfg, seed=rep)
        except pm.ProtocolError as e:
            assert "in flight" in str(e)
            return
    pytest.fail(f"{plant!r} went unnoticed")


PLANTS = {
    "empty_parity": True,           # producer waits the K/V release of the wrong phase
    "no_s_free_wait": True,         # S_0(j+1) issued before the softmax read S_0(j)
    "s1_skips_k_wait": True,        # S_1(j+1) for the extra key tile of a causal unit without K's wait
    "s_skips_k_wait": True,         # a tile issuer (non-causal d <= 64) issues S_i(j+1) without K's wait
    "s_before_pv": False,           # d = 128: S_0(j+1) overwrites P_0(j) before PV_0(j)
    "rescale_before_o_done": True,  # O_i rescaled before PV_i(j-1) completed
    "no_o_done_wait": True,         # P_i(j) written while PV_i(j-1) may still read P_i(j-1)
    "pv_ready_before_rescale": True,   # softmax releases PV_i(j) before rescaling O_i (d <= 64)
    "arrive_before_rescale": False,    # correction releases PV_i(j) before rescaling O_i (d = 128)
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_model_finds_planted_mistakes(plant):
    sep = PLANTS[plant]
    for rep in range(400):
        rng = random.Random(rep)
        causal = rep % 2 == 0
        cfg = pm.Config(separate_p=sep, causal=causal, stages=2 + rep % 3,
                        units=pm.random_units(rng, causal, rng.randint(1, 4)), plant=plant,
                        tma_weight=0.01 if rep % 4 >= 2 else 1.0)   # half the runs: slow TMA loads
        try:
            pm.run(cfg, seed=rep)
        except pm.ProtocolError:
            return
    pytest.fail(f"planted mistake {plant!r} went unnoticed in 400 schedules")


def test_softmax_o_free_wait_is_a_second_guard():
    """One MMA issuer for both tiles (causal d <= 64, and d = 128): the softmax's wait for the
    previous epilogue (o_free) before it publishes a unit's final m, l is implied by the rest of
    the protocol -- the next unit's first S_i is issued only after PV_i(0) of the current unit,
    which waited for the epilogue two units back.  Without the wait the model finds no stale
    read; the kernel keeps it as a second guard."""
    for rep in range(200):
        rng = random.Random(rep)
        sep = rep % 2 == 0
        cfg = pm.Config(separate_p=sep, causal=True, stages=3 if sep else 2,
                        units=pm.random_units(rng, True, rng.randint(2, 6), max_tiles=2),
                        plant="stats_no_o_free_wait")
        pm.run(cfg, seed=rep)


def test_softmax_o_free_wait_is_needed_with_tile_issuers():
    """One MMA issuer per tile (non-causal d <= 64): a tile's issuer does not wait for the other
    tile's PVs, so a softmax warpgroup can run two units ahead of the epilogue, and without the
    o_free wait its statistics overtake the epilogue's reads; the model must find that."""
    for rep in range(400):
        rng = random.Random(rep)
        cfg = pm.Config(separate_p=True, causal=False, stages=3,
                        units=pm.random_units(rng, False, rng.randint(2, 6), max_tiles=2),
                        plant="stats_no_o_free_wait")
        try:
            pm.run(cfg, seed=rep)
        except pm.ProtocolError:
            return
    pytest.fail("the missing o_free wait went unnoticed in 400 schedules")


def test_model_barriers_match_the_kernel_source():
    # The model must know every mbarrier the kernel initialises, with the same arrival count;
    # a barrier added to or re-counted in the kernel without the model fails here.
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "exact_attention_sdpa_b200", "csrc",
                            "attn_fwd_kernel.cuh")).read()
    assert "constexpr bool kTileIssuers = C::kSeparateP && !CAUSAL;" in src
    assert "constexpr uint32_t kReleases = kTileIssuers ? 2 : 1;" in src
    for sep, causal in ((True, True), (True, False), (False, True)):
        found = {}
        for name, expr in re.findall(r"mbar_init\(&sh\.(\w+)(?:\[[^\]]*\])*,\s*([^;]+)\);", src):
            # C::kPvArrivals: the softmax's 128 arrivals, plus the correction's 128 at d = 128;
            # kReleases: one K/V/drain release per MMA issuer
            found[name] = eval(expr.strip().replace("C::kPvArrivals", "kPv"),
                               {"kBlockM": 128, "kPv": 128 if sep else 256, "kReleases": 2 if sep and not causal else 1})
        found.pop("never")            # stall-injection target: nothing ever arrives on it
        check_barriers(found, pm.State(pm.Config(units=[(1, 1)], bias_stages=1, separate_p=sep, causal=causal)))


def check_barriers(found, st):
    model = {}
    for name, val in vars(st).items():
        bars = val
        while isinstance(bars, list) and bars and isinstance(bars[0], list):
            bars = bars[0]
        if isinstance(bars, list) and bars and isinstance(bars[0], pm.Barrier):
            model[name] = bars[0].count
        elif isinstance(val, pm.Barrier):
            model[name] = val.count
    model.pop("teardown")         # the kernel's __syncthreads before tensor memory is freed
    assert found == model
