"""The forward kernel's work decomposition, restated on the CPU and checked over random shapes.

decode_unit (exact_attention_sdpa_b200/csrc/attn_fwd_kernel.cuh) maps a unit index to a
(sequence, head, 256-row query pair) and to the key tiles each of its two 128-row query tiles
visits: tiles [kv_lo, kv_lo + nkv_i).  Causal units stop at the tile holding the last row's
last visible key; with a left window (score modification) the unit starts at the tile holding
its first row's first visible key.  A ragged batch carries a table of sequences (unit prefix
sums, query and key offsets and lengths) and each unit finds its sequence by binary search;
attn_fwd_varlen orders the sequences heaviest first.

The restatement below mirrors that code line by line (a change there must be mirrored here).
The properties checked are the ones the kernel's correctness rests on: every (sequence, head,
query pair) is produced exactly once; every key visible to any row of a query tile lies in the
tile's key range (nothing visible is skipped); each tile visits at least one key tile; and no
visited key tile lies wholly past the last key."""
import random

import pytest

BM = BN = 128
ROWS_PER_UNIT = 256


def decode(u, p):
    """Mirror of decode_unit: returns dict(seq, h, qp, q0, nkv0, nkv1, kv_lo, N, Nk, off)."""
    U = {}
    if p["n_seq"] > 0:
        lo, hi = 0, p["n_seq"] - 1
        while lo < hi:
            mid = (lo + hi + 1) >> 1
            if p["seq_units"][mid] <= u:
                lo = mid
            else:
                hi = mid - 1
        r = u - p["seq_units"][lo]
        s = lo
        if p.get("level_order"):
            per_pair = (lo + 1) * p["H"]
            t, w = r // per_pair, r % per_pair
            s = w // p["H"]
            U["qp"] = (p["seq_nq"][lo] + ROWS_PER_UNIT - 1) // ROWS_PER_UNIT - 1 - t
            U["h"] = w % p["H"]
        else:
            nqp = (p["seq_nq"][lo] + ROWS_PER_UNIT - 1) // ROWS_PER_UNIT
            U["qp"] = nqp - 1 - r // p["H"]
            U["h"] = r % p["H"]
        U["N"], U["Nk"] = p["seq_nq"][s], p["seq_nk"][s]
        U["seq"] = s
    else:
        BH, G = p["B"] * p["H"], p["head_group"]
        per = G * p["num_q_pairs"]
        g, r = u // per, u % per
        gsize = min(G, BH - g * G)
        U["qp"] = p["num_q_pairs"] - 1 - r // gsize
        bh = g * G + r % gsize
        U["seq"], U["h"] = bh // p["H"], bh % p["H"]
        U["N"], U["Nk"] = p["N"], p["Nk"]
    U["off"] = U["Nk"] - U["N"]
    n_kv = (U["Nk"] + BN - 1) // BN
    U["q0"] = U["qp"] * ROWS_PER_UNIT
    if p["causal"]:
        last0 = U["q0"] + BM - 1 + U["off"]
        last1 = last0 + BM
        U["nkv0"] = 1 if last0 < 0 else min(n_kv, last0 // BN + 1)
        U["nkv1"] = 1 if last1 < 0 else min(n_kv, last1 // BN + 1)
    else:
        U["nkv0"] = U["nkv1"] = n_kv
    U["kv_lo"] = 0
    if p.get("mods") and p["window_left"] >= 0:
        lo_key = U["q0"] + U["off"] - p["window_left"]
        U["kv_lo"] = lo_key // BN if lo_key > 0 else 0
        U["nkv0"] -= U["kv_lo"]
        U["nkv1"] -= U["kv_lo"]
    return U


def visible_keys(i, N, Nk, causal, window):
    """Keys row i sees (the oracle's definition): j <= i + Nk - N if causal, j >= i + Nk - N - w."""
    off = Nk - N
    hi = min(Nk - 1, i + off) if causal else Nk - 1
    lo = max(0, i + off - window) if window >= 0 else 0
    return lo, hi


def check_units(p, problems):
    """problems: {seq: (N, Nk)}; asserts the properties for every unit of p."""
    seen = set()
    for u in range(p["num_units"]):
        U = decode(u, p)
        key = (U["seq"], U["h"], U["qp"])
        assert key not in seen, key
        seen.add(key)
        N, Nk = problems[U["seq"]]
        assert (U["N"], U["Nk"]) == (N, Nk)
        assert 0 <= U["qp"] and U["q0"] < N
        for i, nkv in enumerate((U["nkv0"], U["nkv1"])):
            assert nkv >= 1
            first, last = U["kv_lo"] * BN, (U["kv_lo"] + nkv) * BN - 1
            assert U["kv_lo"] * BN < Nk, "a key tile wholly past the last key"
            assert (U["kv_lo"] + nkv - 1) * BN < Nk
            for row in range(U["q0"] + i * BM, min(N, U["q0"] + (i + 1) * BM)):
                lo, hi = visible_keys(row, N, Nk, p["causal"], p["window_left"] if p.get("mods") else -1)
                if lo <= hi:
                    assert first <= lo and hi <= last, (row, lo, hi, first, last)
    want = {(s, h, qp) for s, (N, Nk) in problems.items() for h in range(p["H"])
            for qp in range((N + ROWS_PER_UNIT - 1) // ROWS_PER_UNIT)}
    assert seen == want


def dense_params(B, H, N, Nk, causal, window=-1, head_group=None):
    nqp = (N + ROWS_PER_UNIT - 1) // ROWS_PER_UNIT
    return {"n_seq": 0, "B": B, "H": H, "N": N, "Nk": Nk, "num_q_pairs": nqp, "num_units": nqp * B * H,
            "head_group": head_group or B * H, "causal": causal, "window_left": window, "mods": window >= 0}


@pytest.mark.parametrize("seed", range(40))
def test_dense_problems_with_windows(seed):
    rng = random.Random(seed)
    B, H = rng.randint(1, 3), rng.randint(1, 3)
    N = rng.randint(1, 1500)
    Nk = N if rng.random() < 0.5 else rng.randint(1, 2000)
    causal = rng.random() < 0.7
    window = rng.choice([-1, 0, 1, rng.randint(0, 400), rng.randint(0, 3000)])
    hg = rng.randint(1, B * H)
    problems = {b: (N, Nk) for b in range(B)}
    check_units(dense_params(B, H, N, Nk, causal, window, hg), problems)


def varlen_params(lengths, H, causal):
    """attn_fwd_varlen's table: non-empty sequences heaviest first (query rows x visible keys)."""
    order = [b for b, (nq, nk) in enumerate(lengths) if nq > 0]
    work = lambda b: (lengths[b][0] * (lengths[b][1] - 0.5 * lengths[b][0]) if causal
                      else lengths[b][0] * lengths[b][1])
    order.sort(key=lambda b: -work(b))        # (Python's sort is stable, as std::stable_sort)
    launches = []
    pairs = lambda b: (lengths[b][0] + ROWS_PER_UNIT - 1) // ROWS_PER_UNIT
    for c0 in range(0, len(order), 64):
        chunk = order[c0:c0 + 64]
        # causal with N_q = N_k in every sequence: units ordered by query pair across the chunk
        level = causal and all(lengths[b][0] == lengths[b][1] for b in chunk)
        units, su = 0, []
        for i, b in enumerate(chunk):
            su.append(units)
            if level:
                below = pairs(chunk[i + 1]) if i + 1 < len(chunk) else 0
                units += (i + 1) * H * (pairs(b) - below)
            else:
                units += H * pairs(b)
        su.append(units)
        p = {"n_seq": len(chunk), "H": H, "seq_units": su, "num_units": units, "causal": causal,
             "window_left": -1, "seq_nq": [lengths[b][0] for b in chunk],
             "seq_nk": [lengths[b][1] for b in chunk], "level_order": level}
        launches.append((p, {s: lengths[b] for s, b in enumerate(chunk)}))
    return launches, order


@pytest.mark.parametrize("seed", range(25))
def test_ragged_batches(seed):
    rng = random.Random(100 + seed)
    n = rng.choice([1, 3, 16, 64, 65, 130])
    lengths = []
    for _ in range(n):
        nq = 0 if rng.random() < 0.1 else rng.randint(1, 1300)
        nk = nq if rng.random() < 0.6 else max(1, rng.randint(1, 2000))
        lengths.append((nq, nk))
    H = rng.randint(1, 4)
    causal = rng.random() < 0.7
    launches, order = varlen_params(lengths, H, causal)
    covered = []
    for p, problems in launches:
        check_units(p, problems)
        covered += [p["seq_nq"][s] for s in range(p["n_seq"])]
    assert len(order) == sum(1 for nq, _ in lengths if nq > 0) == len(covered)


def test_planted_mistake_in_the_window_start_is_caught():
    """A window start rounded up instead of down skips visible keys; the check must see it."""
    p = dense_params(1, 1, 1000, 1000, True, window=200)
    bad = dict(p)
    orig = decode

    def decode_round_up(u, q):
        U = orig(u, q)
        lo_key = U["q0"] + U["off"] - q["window_left"]
        if lo_key > 0 and lo_key % BN:
            U["kv_lo"] += 1
            U["nkv0"] -= 1
            U["nkv1"] -= 1
        return U
    globals()["decode"] = decode_round_up
    try:
        with pytest.raises(AssertionError):
            check_units(bad, {0: (1000, 1000)})
    finally:
        globals()["decode"] = orig


@pytest.mark.parametrize("seed", range(20))
def test_ragged_causal_batches_in_query_pair_order(seed):
    """Causal ragged batches with N_q = N_k in every sequence: the launch takes the units of all
    sequences by query pair, highest first -- heaviest first, since a causal pair's key tiles
    depend on its index only -- and still every (sequence, head, pair) exactly once."""
    rng = random.Random(300 + seed)
    n = rng.choice([1, 2, 5, 16, 64, 70])
    lengths = [(m, m) for m in (rng.randint(1, 2500) for _ in range(n))]
    H = rng.randint(1, 4)
    launches, order = varlen_params(lengths, H, True)
    for p, problems in launches:
        assert p["level_order"]
        check_units(p, problems)
        qps = [decode(u, p)["qp"] for u in range(p["num_units"])]
        assert all(a >= b for a, b in zip(qps, qps[1:])), "units not in non-increasing pair order"
        weights = [decode(u, p)["nkv1"] for u in range(p["num_units"])]
        assert all(a >= b for a, b in zip(weights, weights[1:])), "units not heaviest first"
