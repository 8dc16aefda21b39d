"""A model of the forward kernel's mbarrier protocol, checked under random interleavings.

The kernel in exact_attention_sdpa_b200/csrc/attn_fwd_kernel.cuh moves every tile between its
roles (TMA producer, MMA issuer -- one per query tile for non-causal d <= 64 --, two softmax
warpgroups, epilogue warpgroup) through
mbarriers whose waits name a phase only by its parity.  compute-sanitizer cannot run on the
machines these kernels are measured on, so this module re-states the protocol as it is written
in the kernel, one actor per warp, and executes it on the CPU under random schedules:

  * each warp is a generator that yields one action at a time (wait, arrive, tcgen05 issue or
    commit, TMA load, tensor/shared memory read or write);
  * tcgen05 operations run asynchronously: each issuing thread has a FIFO (operations from one
    thread execute in issue order, as the tcgen05 ordering rules state), and a commit arrives on
    its barrier only once everything that thread issued before it has executed.  Operations of
    different threads execute in any order;
  * TMA loads complete in any order and then arrive on their barrier;
  * every buffer (Q, K, V and bias stages in shared memory; S, P, O columns in tensor memory;
    the statistics slots) carries a version tag, and every read checks that it sees
    exactly the version the kernel means to read.

A run fails on a stale or early read (a race), on a wait that returns while its barrier is not
exactly one phase past the phase the waiter means (parity aliasing), on a state where no
actor can move (deadlock), or, when a bounded wait was made to give up (Config.timeout), on a
teardown reached while a TMA load or a tensor-core operation is still in flight.  The model is a restatement of the kernel's control flow, not the
kernel itself: a change to the kernel's barrier protocol has to be mirrored here.
"""
from __future__ import annotations

import random
from dataclasses import dataclass, field


class ProtocolError(AssertionError):
    pass


class Barrier:
    """mbarrier: `count` arrivals complete a phase; try_wait(parity) is true once the phase of
    that parity has completed (so parity 1 reads as complete before anything arrived)."""

    def __init__(self, name: str, count: int):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self, n: int = 1) -> None:
        self.pending -= n
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: {-self.pending} arrivals beyond the count in phase {self.completed}")
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def try_wait(self, parity: int) -> bool:
        return (self.completed & 1) != (parity & 1)


# ---------------------------------------------------------------------------------------- actions
@dataclass
class Wait:
    bar: Barrier
    parity: int
    phase: int          # the phase the waiter means (its completion); parity must equal phase & 1
    drain: bool = False  # a drain wait on exit: ignores the abort flag (the kernel's drain_phase)


@dataclass
class Arrive:
    bar: Barrier
    n: int


@dataclass
class Issue:          # a tcgen05.mma (or any async tensor-core operation) from thread `thread`
    thread: str
    name: str
    run: object       # callable(state) executed when the tensor core performs it


@dataclass
class Commit:         # tcgen05.commit from `thread` onto `bar`
    thread: str
    bar: Barrier


@dataclass
class Tma:            # a TMA load: `run(state)` writes the destination, then one arrival on `bar`
    name: str
    run: object
    bar: Barrier


@dataclass
class Do:             # a synchronous step of the warp itself (tcgen05.ld/st + wait, shared memory)
    name: str
    run: object


# ---------------------------------------------------------------------------------------- config
@dataclass
class Config:
    separate_p: bool = True       # d <= 64: P has its own columns; d = 128: P overwrites S
    causal: bool = True
    stages: int = 3               # K/V ring depth
    bias_stages: int = 0          # staged bias tiles per query tile (0: no bias through TMA)
    units: list = field(default_factory=list)    # per unit (nkv0, nkv1)
    plant: str = ""               # a protocol mistake planted on purpose (tests of the checker)
    timeout: tuple = ()           # (role, n): that role's n-th bounded wait gives up (abort path)
    tma_weight: float = 1.0       # relative chance that a pending TMA load completes next (< 1: slow loads)


def random_units(rng: random.Random, causal: bool, n_units: int, max_tiles: int = 5) -> list:
    out = []
    for _ in range(n_units):
        n0 = rng.randint(1, max_tiles)
        # causal: the second query tile reaches at most one more key tile (its rows are 128 later)
        n1 = n0 + (rng.random() < 0.5) if causal else n0
        out.append((n0, n1))
    return out


def tile_issuers(cfg: "Config") -> bool:
    """The kernel's kTileIssuers: separate P columns (d <= 64) without causal masking."""
    return cfg.separate_p and not cfg.causal


# ---------------------------------------------------------------------------------------- state
class State:
    def __init__(self, cfg: Config):
        self.cfg = cfg
        ST, BS = cfg.stages, max(cfg.bias_stages, 1)
        B = Barrier
        self.q_full = [B(f"q_full{i}", 1) for i in range(2)]
        self.q_empty = [B(f"q_empty{i}", 1) for i in range(2)]
        self.k_full = [B(f"k_full{s}", 1) for s in range(ST)]
        # non-causal d <= 64: one issuer per query tile, each releasing every K / V stage and the
        # drain once
        rel = 2 if tile_issuers(cfg) else 1
        self.k_empty = [B(f"k_empty{s}", rel) for s in range(ST)]
        self.v_full = [B(f"v_full{s}", 1) for s in range(ST)]
        self.v_empty = [B(f"v_empty{s}", rel) for s in range(ST)]
        self.s_full = [B(f"s_full{i}", 1) for i in range(2)]
        self.s_free = [B(f"s_free{i}", 128) for i in range(2)]
        # separate P (d <= 64): the softmax rescales O itself and alone releases PV_i(j); P inside S
        # (d = 128): the correction warpgroup rescales O and releases PV_i(j) with the softmax
        self.pv_ready = [B(f"pv_ready{i}", 128 if cfg.separate_p else 256) for i in range(2)]
        self.o_done = [B(f"o_done{i}", 1) for i in range(2)]
        self.o_final = [B(f"o_final{i}", 1) for i in range(2)]
        self.sm2corr = [B(f"sm2corr{i}", 128) for i in range(2)]
        self.o_free = [B(f"o_free{i}", 128) for i in range(2)]
        self.stats_full = [B(f"stats_full{i}", 128) for i in range(2)]
        self.bias_full = [[B(f"bias_full{i}.{s}", 1) for s in range(BS)] for i in range(2)]
        self.bias_empty = [[B(f"bias_empty{i}.{s}", 128) for s in range(BS)] for i in range(2)]
        self.drain = B("drain", rel)
        # __syncthreads before tensor memory is freed (one arrival per modelled warp)
        self.teardown = B("teardown", 15 if tile_issuers(cfg) else 14)
        self.abort = False                            # the CTA's abort flag
        # buffers (version tags)
        self.sQ = [None, None]
        self.sK = [None] * ST
        self.sV = [None] * ST
        self.sBias = [[None] * BS for _ in range(2)]
        # tensor memory, per query tile and lane quarter (warp q of a warpgroup owns lanes 32q..)
        self.tS = [[None] * 4 for _ in range(2)]      # S_i (and P_i at d = 128)
        self.tP = [[None] * 4 for _ in range(2)]      # P_i (d <= 64)
        self.tO = [[None] * 4 for _ in range(2)]      # O_i: dict(unit, done, rescaled, read)
        self.stats = [[[None] * 4 for _ in range(2)] for _ in range(2)]   # [unit parity][tile][quarter]
        self.alpha = [[[None] * 4 for _ in range(2)] for _ in range(2)]   # [j parity][tile][quarter] (d = 128)

    def expect(self, what: str, got, want) -> None:
        if got != want:
            raise ProtocolError(f"{what}: read {got!r}, expected {want!r}")


# ---------------------------------------------------------------------------------------- roles
# Each role mirrors its branch of the kernel, including what it does when a bounded wait gives
# up: `ok = yield Wait(...)` is False after a timeout or once another role raised the abort flag,
# and the role then leaves its loops the way the kernel does, drains, and meets the others at
# the teardown barrier.

def nkv_of(cfg: Config, k: int, i: int) -> int:
    return cfg.units[k][i]


def teardown(st: State):
    yield Arrive(st.teardown, 1)
    yield Wait(st.teardown, 0, 0, drain=True)


def producer(st: State):
    """TMA producer warp: [bias(0)], Q0, K(0), Q1, V(0), then K(j), V(j), [bias(j)] per unit; drains."""
    cfg, ST, BS = st.cfg, st.cfg.stages, st.cfg.bias_stages
    cnt = {"K": 0, "V": 0}
    qc = [0, 0]
    bc = [0, 0]
    ok = True

    def WU(bar, parity, phase):
        nonlocal ok
        if ok:
            ok = yield Wait(bar, parity, phase)
        return ok

    def load_q(i, k):
        if qc[i] > 0 and not (yield from WU(st.q_empty[i], (qc[i] - 1) & 1, qc[i] - 1)):
            return

        def run(s, i=i, k=k):
            s.sQ[i] = k
        yield Tma(f"Q{i} unit {k}", run, st.q_full[i])
        qc[i] += 1

    def load_kv(kind):
        full, empty, buf = ((st.k_full, st.k_empty, "sK") if kind == "K" else (st.v_full, st.v_empty, "sV"))
        n = cnt[kind]
        s_ = n % ST
        if n >= ST:
            par = (n // ST) & 1 if cfg.plant == "empty_parity" else ((n // ST) - 1) & 1
            if not (yield from WU(empty[s_], par, n // ST - 1)):
                return

        def run(s, s_=s_, tile_id=n):
            getattr(s, buf)[s_] = tile_id
        yield Tma(f"{kind} tile {n}", run, full[s_])
        cnt[kind] += 1

    def load_bias(i, j, k):
        s_ = bc[i] % BS
        if bc[i] >= BS and not (yield from WU(st.bias_empty[i][s_], ((bc[i] // BS) - 1) & 1, bc[i] // BS - 1)):
            return

        def run(s, i=i, s_=s_, j=j, k=k):
            s.sBias[i][s_] = (k, j)
        yield Tma(f"bias{i} ({k},{j})", run, st.bias_full[i][s_])
        bc[i] += 1

    for k, (n0, n1) in enumerate(cfg.units):
        if not ok:
            break
        if BS:                             # the unit's first bias tiles go first
            yield from load_bias(0, 0, k)
            if ok:
                yield from load_bias(1, 0, k)
        if ok:
            yield from load_q(0, k)
        if ok:
            yield from load_kv("K")
        if ok:
            yield from load_q(1, k)
        if ok:
            yield from load_kv("V")
        j = 1
        while ok and j < n1:
            yield from load_kv("K")
            if ok:
                yield from load_kv("V")
            if BS:
                if ok and j < n0:
                    yield from load_bias(0, j, k)
                if ok:
                    yield from load_bias(1, j, k)
            j += 1
    # every load issued into shared memory lands before the CTA exits
    if cfg.plant == "no_tma_drain":
        yield from teardown(st)
        return
    for i in range(2):
        if qc[i] > 0:
            yield Wait(st.q_full[i], (qc[i] - 1) & 1, qc[i] - 1, drain=True)
    for s_ in range(ST):
        for kind, full in (("K", st.k_full), ("V", st.v_full)):
            if cnt[kind] > s_:
                n = (cnt[kind] - 1 - s_) // ST
                yield Wait(full[s_], n & 1, n, drain=True)
    for i in range(2):
        for s_ in range(BS):
            if bc[i] > s_:
                n = (bc[i] - 1 - s_) // BS
                yield Wait(st.bias_full[i][s_], n & 1, n, drain=True)
    yield from teardown(st)


def s_mma(st: State, i: int, k: int, j: int, kst: int, key_tile: int, thread: str = "mma"):
    def run(s):
        s.expect(f"S{i}({k},{j}) reads Q{i}", s.sQ[i], k)
        s.expect(f"S{i}({k},{j}) reads K stage {kst}", s.sK[kst], key_tile)
        for q in range(4):
            s.tS[i][q] = ("S", k, j)
    return Issue(thread, f"S{i}({k},{j})", run)


def pv_mma(st: State, i: int, k: int, j: int, vst: int, key_tile: int, thread: str = "mma"):
    def run(s):
        s.expect(f"PV{i}({k},{j}) reads V stage {vst}", s.sV[vst], key_tile)
        for q in range(4):
            p = s.tP[i][q] if s.cfg.separate_p else s.tS[i][q]
            s.expect(f"PV{i}({k},{j}) reads P{i} lanes {q}", p, ("P", k, j))
            o = s.tO[i][q]
            if j == 0:
                if o is not None and not o["read"]:
                    raise ProtocolError(f"PV{i}({k},0) overwrites O{i} before the epilogue of unit {o['unit']} read it")
            else:
                s.expect(f"PV{i}({k},{j}) accumulates onto O{i}", (o["unit"], o["done"]), (k, j - 1))
                if o["rescaled"] != j:
                    raise ProtocolError(f"PV{i}({k},{j}) runs before O{i} was rescaled for alpha({j})")
            s.tO[i][q] = {"unit": k, "done": j, "rescaled": o["rescaled"] if j else 0, "read": False}
    return Issue(thread, f"PV{i}({k},{j})", run)


def mma_tile_issuer(st: State, ti: int):
    """Non-causal d <= 64: the issuing warp of query tile ti (warp 12 for tile 0, warp 14 for
    tile 1).  S_ti(j+1) as soon as S_ti(j) was read, then PV_ti(j); the next unit's S_ti(0) right
    behind the unit's last PV_ti; one release of every K and V stage it read, one commit to the
    drain.  Both tiles take the same key tiles (no causal masking)."""
    cfg, ST = st.cfg, st.cfg.stages
    thread = f"mma{ti}"
    kc = vc = 0
    pv_n = sf_n = 0
    early = False
    n_units = len(cfg.units)
    ok = True

    def W(bar, parity, phase):
        nonlocal ok
        if ok:
            ok = yield Wait(bar, parity, phase)
        return ok

    def first_s(k, kpos, nkv):
        if not (yield from W(st.q_full[ti], k & 1, k)):
            return False
        if not (yield from W(st.k_full[kpos % ST], (kpos // ST) & 1, kpos // ST)):
            return False
        yield s_mma(st, ti, k, 0, kpos % ST, kpos, thread)
        yield Commit(thread, st.s_full[ti])
        yield Commit(thread, st.k_empty[kpos % ST])
        if nkv == 1:
            yield Commit(thread, st.q_empty[ti])
        return True

    for k in range(n_units):
        nkv = cfg.units[k][ti]
        nkv_next = cfg.units[k + 1][ti] if k + 1 < n_units else 0
        if not ok:
            break
        if not early and not (yield from first_s(k, kc, nkv)):
            break
        early = False
        for j in range(nkv):
            vn, kn = vc + j, kc + j + 1
            vst, vph, kst, kph = vn % ST, (vn // ST) & 1, kn % ST, (kn // ST) & 1
            if j + 1 < nkv:
                if not (cfg.plant == "no_s_free_wait" and ti == 0) and \
                        not (yield from W(st.s_free[ti], sf_n & 1, sf_n)):
                    break
                sf_n += 1
                if cfg.plant != "s_skips_k_wait" and not (yield from W(st.k_full[kst], kph, kn // ST)):
                    break
                yield s_mma(st, ti, k, j + 1, kst, kn, thread)
                yield Commit(thread, st.s_full[ti])
                yield Commit(thread, st.k_empty[kst])
                if j + 2 == nkv:
                    yield Commit(thread, st.q_empty[ti])
            if not (yield from W(st.pv_ready[ti], pv_n & 1, pv_n)):
                break
            pv_n += 1
            if j == 0 and k > 0 and not (yield from W(st.o_free[ti], (k - 1) & 1, k - 1)):
                break
            if not (yield from W(st.v_full[vst], vph, vn // ST)):
                break
            yield pv_mma(st, ti, k, j, vst, vn, thread)
            yield Commit(thread, st.o_done[ti])
            yield Commit(thread, st.v_empty[vst])
            if j + 1 == nkv:
                yield Commit(thread, st.o_final[ti])
                if nkv_next > 0:
                    if not (yield from first_s(k + 1, kc + nkv, nkv_next)):
                        break
                    early = True
        kc += nkv
        vc += nkv
    if cfg.plant != "no_mma_drain":
        yield Commit(thread, st.drain)
        yield Wait(st.drain, 0, 0, drain=True)
    yield from teardown(st)


def mma_issuer(st: State):
    """The single MMA warp (warp 12): S_i(j+1) as soon as S_i(j) was read, then PV_i(j)."""
    cfg, ST = st.cfg, st.cfg.stages
    kc = vc = 0
    pv_cnt, sf_cnt = [0, 0], [0, 0]
    early = [False, False]
    n_units = len(cfg.units)
    ok = True

    def W(bar, parity, phase):
        nonlocal ok
        if ok:
            ok = yield Wait(bar, parity, phase)
        return ok

    def first_s(i, k, kpos, nkv_i):
        if not (yield from W(st.q_full[i], k & 1, k)):
            return False
        if not (yield from W(st.k_full[kpos % ST], (kpos // ST) & 1, kpos // ST)):
            return False
        yield s_mma(st, i, k, 0, kpos % ST, kpos)
        yield Commit("mma", st.s_full[i])
        if i == 1:
            yield Commit("mma", st.k_empty[kpos % ST])
        if nkv_i == 1:
            yield Commit("mma", st.q_empty[i])
        return True

    for k, (n0, n1) in enumerate(cfg.units):
        if not ok:
            break
        nxt = cfg.units[k + 1] if (cfg.separate_p and k + 1 < n_units) else (0, 0)
        if not early[0] and not (yield from first_s(0, k, kc, n0)):
            break
        if not early[1] and not (yield from first_s(1, k, kc, n1)):
            break
        early = [False, False]
        for j in range(n1):
            vn, kn = vc + j, kc + j + 1
            vst, vph, kst, kph = vn % ST, (vn // ST) & 1, kn % ST, (kn // ST) & 1
            if cfg.separate_p:
                if j + 1 < n0:
                    if cfg.plant != "no_s_free_wait" and not (yield from W(st.s_free[0], sf_cnt[0] & 1, sf_cnt[0])):
                        break
                    sf_cnt[0] += 1
                    if not (yield from W(st.k_full[kst], kph, kn // ST)):
                        break
                    yield s_mma(st, 0, k, j + 1, kst, kn)
                    yield Commit("mma", st.s_full[0])
                    if j + 2 == n0:
                        yield Commit("mma", st.q_empty[0])
                if j + 1 < n1:
                    if not (yield from W(st.s_free[1], sf_cnt[1] & 1, sf_cnt[1])):
                        break
                    sf_cnt[1] += 1
                    if j + 1 >= n0 and cfg.plant != "s1_skips_k_wait" and not (yield from W(st.k_full[kst], kph, kn // ST)):
                        break
                    yield s_mma(st, 1, k, j + 1, kst, kn)
                    yield Commit("mma", st.s_full[1])
                    yield Commit("mma", st.k_empty[kst])
                    if j + 2 == n1:
                        yield Commit("mma", st.q_empty[1])
                if j < n0:
                    if not (yield from W(st.pv_ready[0], pv_cnt[0] & 1, pv_cnt[0])):
                        break
                    pv_cnt[0] += 1
                    if j == 0 and k > 0 and not (yield from W(st.o_free[0], (k - 1) & 1, k - 1)):
                        break
                    if not (yield from W(st.v_full[vst], vph, vn // ST)):
                        break
                    yield pv_mma(st, 0, k, j, vst, vn)
                    yield Commit("mma", st.o_done[0])
                    if j + 1 == n0:
                        yield Commit("mma", st.o_final[0])
                    if j + 1 == n0 and nxt[0] > 0:
                        if not (yield from first_s(0, k + 1, kc + n1, nxt[0])):
                            break
                        early[0] = True
                if not (yield from W(st.pv_ready[1], pv_cnt[1] & 1, pv_cnt[1])):
                    break
                pv_cnt[1] += 1
                if j == 0 and k > 0 and not (yield from W(st.o_free[1], (k - 1) & 1, k - 1)):
                    break
                if j >= n0 and not (yield from W(st.v_full[vst], vph, vn // ST)):
                    break
                yield pv_mma(st, 1, k, j, vst, vn)
                yield Commit("mma", st.o_done[1])
                yield Commit("mma", st.v_empty[vst])
                if j + 1 == n1:
                    yield Commit("mma", st.o_final[1])
                if j + 1 == n1 and nxt[1] > 0:
                    if not (yield from first_s(1, k + 1, kc + n1, nxt[1])):
                        break
                    early[1] = True
                continue
            # d = 128: P_i(j) lives in S_i, so S_i(j+1) is issued behind PV_i(j)
            if cfg.plant == "s_before_pv" and j + 1 < n0:
                if not (yield from W(st.k_full[kst], kph, kn // ST)):
                    break
                yield s_mma(st, 0, k, j + 1, kst, kn)
            if j < n0:
                if not (yield from W(st.pv_ready[0], pv_cnt[0] & 1, pv_cnt[0])):
                    break
                pv_cnt[0] += 1
                if j == 0 and k > 0 and not (yield from W(st.o_free[0], (k - 1) & 1, k - 1)):
                    break
                if not (yield from W(st.v_full[vst], vph, vn // ST)):
                    break
                yield pv_mma(st, 0, k, j, vst, vn)
                yield Commit("mma", st.o_done[0])
            if j + 1 < n0:
                if cfg.plant != "s_before_pv":
                    if not (yield from W(st.k_full[kst], kph, kn // ST)):
                        break
                    yield s_mma(st, 0, k, j + 1, kst, kn)
                yield Commit("mma", st.s_full[0])
                if j + 2 == n0:
                    yield Commit("mma", st.q_empty[0])
            if not (yield from W(st.pv_ready[1], pv_cnt[1] & 1, pv_cnt[1])):
                break
            pv_cnt[1] += 1
            if j == 0 and k > 0 and not (yield from W(st.o_free[1], (k - 1) & 1, k - 1)):
                break
            if not (yield from W(st.v_full[vst], vph, vn // ST)):
                break
            yield pv_mma(st, 1, k, j, vst, vn)
            yield Commit("mma", st.o_done[1])
            yield Commit("mma", st.v_empty[vst])
            if j + 1 < n1:
                if not (yield from W(st.k_full[kst], kph, kn // ST)):
                    break
                yield s_mma(st, 1, k, j + 1, kst, kn)
                yield Commit("mma", st.s_full[1])
                yield Commit("mma", st.k_empty[kst])
                if j + 2 == n1:
                    yield Commit("mma", st.q_empty[1])
        kc += n1
        vc += n1
    # all MMAs complete before tensor memory is released
    if cfg.plant != "no_mma_drain":
        yield Commit("mma", st.drain)
        yield Wait(st.drain, 0, 0, drain=True)
    yield from teardown(st)


def softmax_warp(st: State, i: int, q: int):
    """Warp q of softmax warpgroup i: rows 32q..32q+31 of query tile i."""
    cfg, BS = st.cfg, st.cfg.bias_stages
    s_cnt = od_cnt = bcnt = 0
    ok = True
    for k in range(len(cfg.units)):
        if not ok:
            break
        nkv = nkv_of(cfg, k, i)
        for j in range(nkv):
            ok = yield Wait(st.s_full[i], s_cnt & 1, s_cnt)
            s_cnt += 1
            if not ok:
                break

            def read_s(s, k=k, j=j):
                s.expect(f"softmax{i}.{q} reads S{i}({k},{j})", s.tS[i][q], ("S", k, j))
            yield Do("ld S", read_s)
            if cfg.separate_p and j + 1 < nkv:
                yield Arrive(st.s_free[i], 32)
            if BS:
                bst = bcnt % BS
                ok = yield Wait(st.bias_full[i][bst], (bcnt // BS) & 1, bcnt // BS)
                if not ok:
                    break

                def read_b(s, k=k, j=j, bst=bst):
                    s.expect(f"softmax{i}.{q} reads bias", s.sBias[i][bst], (k, j))
                yield Do("read bias", read_b)
                yield Arrive(st.bias_empty[i][bst], 32)
                bcnt += 1

            if not cfg.separate_p and j > 0:
                # d = 128: alpha(j) for the correction (S_i(j) was issued after PV_i(j-1), so the
                # correction has consumed alpha(j-1))
                def put_alpha(s, k=k, j=j):
                    s.alpha[j & 1][i][q] = (k, j)
                yield Do("alpha", put_alpha)
                yield Arrive(st.sm2corr[i], 32)
            if cfg.separate_p and j > 0 and cfg.plant != "rescale_before_o_done":
                # P_i(j) overwrites P_i(j-1) and O_i may be rescaled: PV_i(j-1) must be complete
                if cfg.plant != "no_o_done_wait":
                    ok = yield Wait(st.o_done[i], od_cnt & 1, od_cnt)
                od_cnt += 1

            def rescale(s, k=k, j=j):
                o = s.tO[i][q]
                s.expect(f"softmax{i}.{q} rescales O{i}", None if o is None else (o["unit"], o["done"]), (k, j - 1))
                o["rescaled"] = j

            def write_p(s, k=k, j=j):
                if s.cfg.separate_p:
                    s.tP[i][q] = ("P", k, j)
                else:
                    s.tS[i][q] = ("P", k, j)
            if not ok:
                break
            if cfg.plant == "pv_ready_before_rescale" and j > 0 and cfg.separate_p:
                yield Arrive(st.pv_ready[i], 32)
            if j > 0 and cfg.separate_p:
                yield Do("rescale O", rescale)
            if cfg.separate_p and j > 0 and cfg.plant == "rescale_before_o_done":
                ok = yield Wait(st.o_done[i], od_cnt & 1, od_cnt)
                od_cnt += 1
                if not ok:
                    break
            yield Do("st P", write_p)
            if cfg.plant == "pv_ready_before_rescale" and j > 0 and cfg.separate_p:
                continue
            yield Arrive(st.pv_ready[i], 32)
        if not ok:
            break
        if cfg.separate_p:
            od_cnt += 1
        if k > 0 and cfg.plant != "stats_no_o_free_wait":
            ok = yield Wait(st.o_free[i], (k - 1) & 1, k - 1)
            if not ok:
                break

        def put_stats(s, k=k):
            s.stats[k & 1][i][q] = k
        yield Do("stats", put_stats)
        yield Arrive(st.stats_full[i], 32)
    yield from teardown(st)


def epilogue_warp(st: State, q: int):
    """Warp q of warpgroup 2.  With separate P (d <= 64) the epilogue alone: per unit and tile the
    final statistics and the last PV_i (o_final), then O_i is read and released.  At d = 128 also
    the correction: O_i rescaled for alpha(j) between PV_i(j-1) and PV_i(j), its pv_ready
    arrivals, and the epilogue on o_done's last phase."""
    cfg = st.cfg
    st_cnt, of_cnt, c_cnt = [0, 0], [0, 0], [0, 0]
    n_units = len(cfg.units)
    ok = True

    def WS(bar, counters, i):
        nonlocal ok
        if ok:
            ok = yield Wait(bar, counters[i] & 1, counters[i])
        counters[i] += 1
        return ok

    for k, (n0, n1) in enumerate(cfg.units):
        if not ok:
            break
        if not cfg.separate_p:
            j = 0
            while ok and j < n1:
                for i in range(2):
                    if j >= (n1 if i else n0):
                        continue
                    if j > 0:
                        if not (yield from WS(st.sm2corr[i], c_cnt, i)):
                            break

                        def read_alpha(s, k=k, j=j, i=i):
                            s.expect(f"correction.{q} reads alpha{i}", s.alpha[j & 1][i][q], (k, j))
                        yield Do("alpha", read_alpha)
                        if not (yield from WS(st.o_done[i], of_cnt, i)):
                            break

                        def rescale(s, k=k, j=j, i=i):
                            o = s.tO[i][q]
                            s.expect(f"correction.{q} rescales O{i}", (o["unit"], o["done"]), (k, j - 1))
                            o["rescaled"] = j
                        if cfg.plant == "arrive_before_rescale":
                            yield Arrive(st.pv_ready[i], 32)
                        yield Do("rescale O", rescale)
                        if cfg.plant != "arrive_before_rescale":
                            yield Arrive(st.pv_ready[i], 32)
                    elif k == 0:
                        yield Arrive(st.pv_ready[i], 32)
                j += 1
            if not ok:
                break
        has_next = k + 1 < n_units and not cfg.separate_p
        for i in range(2):
            if not (yield from WS(st.stats_full[i], st_cnt, i)):
                break
            if not (yield from WS(st.o_final[i] if cfg.separate_p else st.o_done[i], of_cnt, i)):
                break
            last = (n1 if i else n0) - 1

            def epilogue(s, k=k, i=i, last=last):
                s.expect(f"epilogue.{q} reads stats{i}", s.stats[k & 1][i][q], k)
                o = s.tO[i][q]
                s.expect(f"epilogue.{q} reads O{i}", (o["unit"], o["done"]), (k, last))
                o["read"] = True
            yield Do("epilogue", epilogue)
            yield Arrive(st.o_free[i], 32)
            if has_next:
                yield Arrive(st.pv_ready[i], 32)
    yield from teardown(st)


def kernel_roles(st: State) -> dict:
    roles = {"tma": producer(st)}
    if tile_issuers(st.cfg):
        roles["mma0"] = mma_tile_issuer(st, 0)
        roles["mma1"] = mma_tile_issuer(st, 1)
    else:
        roles["mma"] = mma_issuer(st)
    for i in range(2):
        for q in range(4):
            roles[f"softmax{i}.{q}"] = softmax_warp(st, i, q)
    for q in range(4):
        roles[f"epi.{q}"] = epilogue_warp(st, q)
    return roles


# ---------------------------------------------------------------------------------------- scheduler
def run(cfg: Config, seed: int, make_roles=kernel_roles, state_cls=State, max_steps: int = 2_000_000,
        info: dict = None) -> int:
    """Executes the roles under one random schedule; returns the number of actions taken.

    A bounded wait (not a drain) returns True once its phase has completed; it returns False
    (leaving the phase unobserved) when the abort flag is up and the phase has not completed,
    or when it is the wait named by cfg.timeout, which also raises the flag.  Drain waits only
    return once their phase completed.  When the teardown barrier completes, no TMA load and no
    tensor-core operation may still be in flight."""
    rng = random.Random(seed)
    st = state_cls(cfg)
    roles = make_roles(st)
    current = {}                    # role -> pending action
    bounded_waits = {}              # role -> bounded waits reached so far
    for name, gen in roles.items():
        current[name] = next(gen, None)
        bounded_waits[name] = 0
    fifos: dict[str, list] = {}     # tcgen05 thread -> [Issue | Commit]
    tma: list = []
    trace: list = []

    def fail(msg):
        tail = "\n  ".join(trace[-25:])
        raise ProtocolError(f"{msg}\n  seed {seed}, units {cfg.units}\n  last actions:\n  {tail}")

    def timed_out(name, a):
        return (not a.drain) and cfg.timeout == (name, bounded_waits[name])

    steps = 0
    while True:
        choices = []
        for name, a in current.items():
            if a is None:
                continue
            if isinstance(a, Wait) and not a.bar.try_wait(a.parity):
                if a.drain or not (st.abort or timed_out(name, a)):
                    continue
            choices.append(("role", name))
        for th, f in fifos.items():
            if f:
                choices.append(("tc", th))
        for idx in range(len(tma)):
            choices.append(("tma", idx))
        if not choices:
            blocked = {n: a for n, a in current.items() if a is not None}
            if blocked:
                desc = ", ".join(f"{n} waits {a.bar.name} phase {a.phase} (completed {a.bar.completed})"
                                 for n, a in blocked.items())
                fail(f"deadlock: {desc}")
            if info is not None:
                info["aborted"] = st.abort
            return steps
        slow = getattr(cfg, "slow_roles", ())     # roles that move rarely (late warps)
        if cfg.tma_weight != 1.0 or slow:
            weights = [cfg.tma_weight if c[0] == "tma" else (0.02 if c[0] == "role" and c[1] in slow else 1.0)
                       for c in choices]
            kind, key = rng.choices(choices, weights)[0]
        else:
            kind, key = rng.choice(choices)
        steps += 1
        if steps > max_steps:
            fail("step limit")
        result = None
        try:
            if kind == "tc":
                item = fifos[key].pop(0)
                if isinstance(item, Issue):
                    trace.append(f"tensor core: {item.name}")
                    item.run(st)
                else:
                    trace.append(f"tensor core: commit -> {item.bar.name}")
                    item.bar.arrive(1)
                continue
            if kind == "tma":
                op = tma.pop(key)
                trace.append(f"TMA done: {op.name}")
                op.run(st)
                op.bar.arrive(1)
                continue
            a = current[key]
            if isinstance(a, Wait):
                if a.parity & 1 != a.phase & 1:
                    fail(f"{key}: waits {a.bar.name} with parity {a.parity} for phase {a.phase}")
                forced = timed_out(key, a)
                if not a.drain:
                    bounded_waits[key] += 1
                if forced or not a.bar.try_wait(a.parity):
                    st.abort = True
                    result = False
                    trace.append(f"{key}: wait on {a.bar.name} phase {a.phase} gives up")
                else:
                    if a.bar.completed != a.phase + 1:
                        fail(f"{key}: wait on {a.bar.name} for phase {a.phase} returned with "
                             f"{a.bar.completed} phases completed (parity aliasing)")
                    result = True
                    trace.append(f"{key}: waited {a.bar.name} phase {a.phase}")
                    if a.bar is st.teardown and (any(fifos.values()) or tma):
                        pending = [i.name if isinstance(i, Issue) else "commit " + i.bar.name
                                   for f in fifos.values() for i in f] + [t.name for t in tma]
                        fail(f"teardown with asynchronous work in flight: {pending}")
            elif isinstance(a, Arrive):
                trace.append(f"{key}: arrive {a.bar.name} x{a.n}")
                a.bar.arrive(a.n)
            elif isinstance(a, (Issue, Commit)):
                fifos.setdefault(a.thread, []).append(a)
                trace.append(f"{key}: issue {a.name if isinstance(a, Issue) else 'commit ' + a.bar.name}")
            elif isinstance(a, Tma):
                tma.append(a)
                trace.append(f"{key}: TMA {a.name}")
            elif isinstance(a, Do):
                trace.append(f"{key}: {a.name}")
                a.run(st)
            else:
                fail(f"{key}: unknown action {a!r}")
        except ProtocolError as e:
            if "last actions" in str(e):
                raise
            fail(str(e))
        try:
            current[key] = roles[key].send(result)
        except StopIteration:
            current[key] = None
