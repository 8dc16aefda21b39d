"""The gradient kernels' mbarrier protocol, restated for the checker in protocol_model.

Both gradient kernels of exact_attention_sdpa_b200/csrc/attn_bwd_tc.cuh (dK/dV and dQ) run one
protocol over a CTA's 128-row block and its nit column blocks:

  * the TMA producer loads the row block's operands (row_full), then column block m into stage
    m % ST (full[s]) once the accumulating products of block m - ST released it (empty[s]);
  * the issuing warp runs products(m) (S and dP, or their transposes) into column set
    m % SETS (SETS = 2 or 3) and commits s_full[set]: first for blocks 0 .. SETS-1, then, per
    block m, after group m % 2's 128 threads arrived on p_ready[set], accumulate(m), a commit
    on empty[s] and products(m + SETS) into the set block m used; a final commit on acc_done
    covers everything, and the warp waits for it before the teardown;
  * each warp of the two elementwise groups, per block of its parity: [dK/dV: warps 0-1 write
    the block's lse and D into the group's buffer it % 2], the group barrier (bar.red.and over
    the group's 128 threads, unbounded), the bounded wait on its block's s_full, the read of the products and
    the store of the 16-bit operands over them, one arrival on the set's p_ready; then the epilogue after
    the bounded acc_done wait (dQ: group g stores 32-column chunks g, g + 2, ...; chunk 0 holds
    the D value the dQ groups read before their first block).

dQ only: the products take Q and dO from tensor memory (TS form).  Each group warp waits for
the row block's TMA load (row_full), copies its rows of Q (group 0) or dO (group 1) from
shared into tensor memory and arrives on row_tmem (256 arrivals); the issuer waits for
row_tmem instead of row_full.

Version tags: the products in a column set are ("prod", m) and, once a warp stored its
operands, ("ops", m); the accumulators count the blocks accumulated; a stage holds the column
block loaded into it; the lse/D buffer holds the block it was written for; the dQ row's chunk
0 holds "D" until a group stores "dQ" over it.
"""
from __future__ import annotations

from dataclasses import dataclass

from protocol_model import Arrive, Barrier, Commit, Do, Issue, ProtocolError, Tma, Wait, run  # noqa: F401

GROUP_WARPS = 4


@dataclass
class BwdConfig:
    kind: str = "dkdv"           # "dkdv" or "dq"
    nit: int = 4                 # column blocks of the CTA
    stages: int = 4              # operand ring depth
    d: int = 64                  # head dim (dQ: the number of 32-column chunks is d / 32)
    sets: int = 2                # product column sets (3 where tensor memory holds them)
    plant: str = ""              # a protocol mistake planted on purpose (tests of the checker)
    timeout: tuple = ()          # (role, n): that role's n-th bounded wait gives up
    tma_weight: float = 1.0
    slow_roles: tuple = ()       # roles the scheduler picks rarely (late warps)
    units: tuple = ()            # unused (the checker prints it on failure)


class BwdState:
    def __init__(self, cfg: BwdConfig):
        self.cfg = cfg
        B, ST = Barrier, cfg.stages
        self.row_full = B("row_full", 1)
        self.row_tmem = B("row_tmem", 128 * 2)
        self.full = [B(f"full{s}", 1) for s in range(ST)]
        self.empty = [B(f"empty{s}", 1) for s in range(ST)]
        self.s_full = [B(f"s_full{c}", 1) for c in range(cfg.sets)]
        self.p_ready = [B(f"p_ready{c}", 128) for c in range(cfg.sets)]
        self.acc_done = B("acc_done", 1)
        self.group_bar = [B(f"group_bar{g}", GROUP_WARPS) for g in range(2)]
        self.teardown = B("teardown", 2 + 2 * GROUP_WARPS)   # __syncthreads before the dealloc
        self.abort = False
        self.votes = [dict(), dict()]          # [group][barrier use] -> AND of the warps' flags
        # buffers
        self.s_row = None
        self.t_row = [[None] * GROUP_WARPS for _ in range(2)]    # dQ: [group][lane quarter] of Q / dO
        self.s_col = [None] * ST
        self.t_set = [[None] * GROUP_WARPS for _ in range(cfg.sets)]   # [column set][lane quarter]
        self.acc = 0
        self.lse_buf = [[None, None] for _ in range(2)]         # [group][buffer]
        self.dq_chunk0 = ["D"] * GROUP_WARPS                    # per lane quarter (row slice)

    def expect(self, what, got, want):
        if got != want:
            raise ProtocolError(f"{what}: read {got!r}, expected {want!r}")


def teardown(st):
    yield Arrive(st.teardown, 1)
    yield Wait(st.teardown, 0, 0, drain=True)


def producer(st: BwdState):
    cfg, ST = st.cfg, st.cfg.stages
    if cfg.nit > 0:
        def row(s):
            s.s_row = "row"
        yield Tma("row block", row, st.row_full)
        issued = [0] * ST
        for m in range(cfg.nit):
            s_, use = m % ST, m // ST
            if use > 0:
                par = use & 1 if cfg.plant == "empty_parity" else (use - 1) & 1
                ok = yield Wait(st.empty[s_], par, use - 1)
                if not ok:
                    break

            def col(s, s_=s_, m=m):
                s.s_col[s_] = m
            yield Tma(f"column block {m}", col, st.full[s_])
            issued[s_] = use + 1
        if cfg.plant != "no_tma_drain":
            yield Wait(st.row_full, 0, 0, drain=True)
            for s_ in range(ST):
                if issued[s_] > 0:
                    yield Wait(st.full[s_], (issued[s_] - 1) & 1, issued[s_] - 1, drain=True)
    yield from teardown(st)


def issuer(st: BwdState):
    cfg, ST, SETS = st.cfg, st.cfg.stages, st.cfg.sets
    nit = cfg.nit
    if nit > 0:
        def products(m):
            s_, c = m % ST, m % SETS

            def run_(s, m=m, s_=s_, c=c):
                if s.cfg.kind == "dq":
                    for g in range(2):
                        for q in range(GROUP_WARPS):
                            s.expect(f"row operand {g} in tensor memory, quarter {q}", s.t_row[g][q], "row")
                else:
                    s.expect("row operands", s.s_row, "row")
                s.expect(f"stage {s_} for products({m})", s.s_col[s_], m)
                for q in range(GROUP_WARPS):
                    s.t_set[c][q] = ("prod", m)
            ok = yield Wait(st.full[s_], (m // ST) & 1, m // ST)
            if not ok:
                return False
            yield Issue("mma", f"products({m})", run_)
            yield Commit("mma", st.s_full[c])
            return True

        def accumulate(m):
            s_, c = m % ST, m % SETS

            def run_(s, m=m, s_=s_, c=c):
                for q in range(GROUP_WARPS):
                    s.expect(f"set {c} operands for accumulate({m})", s.t_set[c][q], ("ops", m))
                s.expect(f"stage {s_} for accumulate({m})", s.s_col[s_], m)
                s.expect("accumulated blocks", s.acc, m)
                s.acc = m + 1
            yield Issue("mma", f"accumulate({m})", run_)
            yield Commit("mma", st.empty[s_])

        if cfg.kind == "dq" and cfg.plant != "mma_skips_row_tmem":
            ok = yield Wait(st.row_tmem, 0, 0)
        elif cfg.kind == "dq":
            ok = True
        else:
            ok = yield Wait(st.row_full, 0, 0)
        m = 0
        while ok and m < SETS and m < nit:
            ok = yield from products(m)
            m += 1
        m = 0
        while ok and m < nit:
            if cfg.plant == "prod_before_acc" and m + SETS < nit:
                ok = yield from products(m + SETS)
                if not ok:
                    break
            if cfg.plant == "p_ready_per_group":
                ok = yield Wait(st.p_ready[m & 1], (m >> 1) & 1, m >> 1)
            else:
                ok = yield Wait(st.p_ready[m % SETS], (m // SETS) & 1, m // SETS)
            if not ok:
                break
            yield from accumulate(m)
            if m + SETS < nit and cfg.plant != "prod_before_acc":
                ok = yield from products(m + SETS)
            m += 1
        yield Commit("mma", st.acc_done)
        if cfg.plant != "no_mma_drain":
            yield Wait(st.acc_done, 0, 0, drain=True)
    yield from teardown(st)


def group_warp(st: BwdState, g: int, q: int):
    cfg = st.cfg
    nit = cfg.nit
    dkdv = cfg.kind == "dkdv"
    reads_d = (g < nit) if cfg.plant != "dq_reads_d_without_block" else (nit > 0)
    if not dkdv and reads_d:
        def read_d(s, q=q):
            s.expect(f"D of quarter {q}", s.dq_chunk0[q], "D")
        yield Do(f"read D (quarter {q})", read_d)
    ok = True
    if not dkdv and nit > 0:
        # the row block's operand into tensor memory (TS products)
        if cfg.plant != "copy_without_row_full":
            ok = yield Wait(st.row_full, 0, 0)
        if ok:
            def copy(s, q=q):
                s.expect(f"row block in shared memory (quarter {q})", s.s_row, "row")
                s.t_row[g][q] = "row"
            yield Do(f"copy row operand {g} (quarter {q})", copy)
            yield Arrive(st.row_tmem, 32)
    it = 0
    for m in range(g, nit, 2):
        buf = 0 if cfg.plant == "lse_single_buffer" else it & 1
        if dkdv and q < 2:                      # threads 0-63 of the group: warps 0 and 1
            def write_l(s, buf=buf, m=m, q=q):
                s.lse_buf[g][buf] = _merge(s.lse_buf[g][buf], q, m)
            yield Do(f"write lse/D of block {m} (half {q})", write_l)
        # group barrier with the AND of the warps' flags
        k = it

        def vote(s, k=k, ok=ok):
            s.votes[g][k] = s.votes[g].get(k, True) and ok
        yield Do(f"group {g} vote {ok}", vote)
        yield Arrive(st.group_bar[g], 1)
        yield Wait(st.group_bar[g], k & 1, k, drain=True)
        ok = st.votes[g][k]
        if not ok:
            break
        c = m % cfg.sets
        if cfg.plant != "no_s_full_wait":
            ok = yield Wait(st.s_full[c], (m // cfg.sets) & 1, m // cfg.sets)
        if ok:
            if dkdv:
                def read_l(s, buf=buf, m=m):
                    s.expect(f"group {g} lse/D buffer {buf}", s.lse_buf[g][buf], (m, m))
                yield Do(f"read lse/D of block {m}", read_l)

            def work(s, m=m, q=q, c=c):
                s.expect(f"set {c} products, quarter {q}", s.t_set[c][q], ("prod", m))
                s.t_set[c][q] = ("ops", m)
            yield Do(f"operands of block {m}", work)
            yield Arrive(st.p_ready[g if cfg.plant == "p_ready_per_group" else c], 32)
        it += 1
    # epilogue
    store = ok and (nit == 0 or (yield Wait(st.acc_done, 0, 0)))
    if store:
        if nit > 0:
            def read_acc(s):
                # (after a timeout the stored gradients are partial; the status word reports it)
                if not s.abort:
                    s.expect("accumulators", s.acc, nit)
            yield Do("read accumulators", read_acc)
        if not dkdv and g == 0:                 # chunk 0 (with D) is group 0's

            def write_dq(s, q=q):
                s.dq_chunk0[q] = "dQ"
            yield Do(f"store dQ chunk 0 (quarter {q})", write_dq)
    yield from teardown(st)


def _merge(cur, q, m):
    """Warps 0 and 1 each write half of the 64 lse/D entries; the buffer reads (m, m) once both
    halves belong to block m."""
    a, b = (cur if cur else (None, None))
    return (m, b) if q == 0 else (a, m)


def bwd_roles(st: BwdState) -> dict:
    roles = {"tma": producer(st), "mma": issuer(st)}
    for g in range(2):
        for q in range(GROUP_WARPS):
            roles[f"grp{g}.{q}"] = group_warp(st, g, q)
    return roles


def run_bwd(cfg: BwdConfig, seed: int, info: dict = None) -> int:
    return run(cfg, seed, make_roles=bwd_roles, state_cls=BwdState, info=info)
