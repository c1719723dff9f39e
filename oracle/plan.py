"""Partition maps and closed-form accounting of the ZeRO step (oracle side).

Test infrastructure only.  Plain Python integers and Fractions, written from
the definitions; shares no code with the library's planner.

Definitions (notation of the pages: Psi parameters, Nd data-parallel ranks,
K bytes of optimizer state per parameter):

* Sharding.  Mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐",
  four-GPU example: the training state is cut into blocks A, B, C, D and GPU i
  keeps block i.  The same page, section "但 GPU 只存四分之一…": each card keeps
  one shard *of the current layer*.  So every unit (a layer, or the whole flat
  vector when there is one unit) is cut into Nd equal contiguous shards and
  rank r owns shard r.  The pages do not say how a length that Nd does not
  divide is handled; the reading taken: each unit is zero-padded to a
  multiple of Nd*A (A = align_elems).
* Buckets.  Concept page "ZeRO", section "关键设计取舍" item 1: large buckets
  use the network better but hold more temporary memory, small ones are
  dominated by launch latency.  Reading taken: a bucket is a contiguous range
  of bucket_elems padded elements of the flat vector, cut at unit boundaries
  (the last bucket of a unit is short).
* Memory per rank.  Mind-map page, section "Stage 1、2、3 不是三套算法…" and
  "论文证据": for 7.5B parameters and Nd = 64 the paper estimates 120 GB for
  plain data parallelism, then 31.4, 16.6 and 1.9 GB as optimizer states,
  gradients and parameters are sharded in turn.  Concept page table "三个阶段"
  says which states are sharded at each stage.  With 2-byte parameters and
  gradients and K = 12 (fp32 master, m, v) the per-rank bytes are
  (2+2+K)Psi, 4Psi + K Psi/Nd, 2Psi + (2+K)Psi/Nd and (2+2+K)Psi/Nd.
* Communication.  Mind-map page, "论文证据": plain data parallelism and
  gradient partitioning move 2Psi per step, parameter partitioning 3Psi,
  about 1.5 times as much.  Reading taken: ring collectives; a reduce-scatter
  or all-gather sends (Nd-1)*S elements per rank (S = elements one rank
  owns); stages 0-2 do one reduce-scatter and one all-gather (an all-reduce is
  the two), stage 3 adds a second all-gather (forward and backward), so
  2(Nd-1)S and 3(Nd-1)S; both tend to 2Psi and 3Psi as Nd grows.
"""
from dataclasses import dataclass, field
from fractions import Fraction
from typing import List, Optional, Tuple


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


@dataclass
class Plan:
    psi: int
    nd: int
    stage: int
    bucket_elems: int
    align: int
    k_bytes: int
    unit_len: List[int]
    unit_pad: List[int] = field(default_factory=list)     # P_u
    unit_shard: List[int] = field(default_factory=list)   # s_u = P_u / Nd
    unit_base: List[int] = field(default_factory=list)    # U_u, logical start
    unit_offset: List[int] = field(default_factory=list)  # O_u, in owner's S
    psi_pad: int = 0
    S: int = 0
    buckets: List[Tuple[int, int, int]] = field(default_factory=list)
    # (unit, logical begin, logical end)


def make_plan(psi: int, nd: int, stage: int, bucket_elems: int, align: int = 64,
              k_bytes: int = 12, unit_elems: Optional[List[int]] = None) -> Plan:
    units = list(unit_elems) if unit_elems else [psi]
    if psi <= 0 or nd <= 0 or align <= 0 or bucket_elems <= 0:
        raise ValueError("psi, nd, align and bucket_elems must be positive")
    if stage not in (0, 1, 2, 3):
        raise ValueError("stage must be 0..3")
    if sum(units) != psi or any(u <= 0 for u in units):
        raise ValueError("unit lengths must be positive and sum to psi")
    pl = Plan(psi, nd, stage, bucket_elems, align, k_bytes, units)
    U = O = 0
    for n in units:
        P = ceil_div(n, nd * align) * nd * align
        s = P // nd
        pl.unit_pad.append(P)
        pl.unit_shard.append(s)
        pl.unit_base.append(U)
        pl.unit_offset.append(O)
        U += P
        O += s
    pl.psi_pad = U
    pl.S = O
    for u, P in enumerate(pl.unit_pad):
        b = 0
        while b < P:
            e = min(b + bucket_elems, P)
            pl.buckets.append((u, pl.unit_base[u] + b, pl.unit_base[u] + e))
            b = e
    return pl


def locate(pl: Plan, p: int) -> Tuple[int, int, int, int]:
    """Logical padded index p -> (unit, owner rank, offset in owner's S block,
    index within the unit); the storage index of p is owner*S + offset."""
    if not 0 <= p < pl.psi_pad:
        raise IndexError(p)
    for u in range(len(pl.unit_pad)):
        if pl.unit_base[u] <= p < pl.unit_base[u] + pl.unit_pad[u]:
            j = p - pl.unit_base[u]
            owner = j // pl.unit_shard[u]
            off = pl.unit_offset[u] + (j - owner * pl.unit_shard[u])
            return u, owner, off, j
    raise AssertionError("unreachable")


def is_padding(pl: Plan, p: int) -> bool:
    u, _, _, j = locate(pl, p)
    return j >= pl.unit_len[u]


def owner_ranges(pl: Plan, rank: int) -> List[Tuple[int, int]]:
    """Logical [begin, end) ranges that `rank` owns, one per unit."""
    out = []
    for u in range(len(pl.unit_pad)):
        b = pl.unit_base[u] + rank * pl.unit_shard[u]
        out.append((b, b + pl.unit_shard[u]))
    return out


# ---------------------------------------------------------------- memory
def memory_bytes_per_rank(stage: int, psi, nd: int, k_bytes: int = 12):
    """Model-state bytes one rank keeps resident (Fraction; unpadded Psi)."""
    psi = Fraction(psi)
    if stage == 0:
        return (2 + 2 + k_bytes) * psi
    if stage == 1:
        return 4 * psi + Fraction(k_bytes) * psi / nd
    if stage == 2:
        return 2 * psi + Fraction(2 + k_bytes) * psi / nd
    if stage == 3:
        return Fraction(2 + 2 + k_bytes) * psi / nd
    raise ValueError(stage)


def memory_bytes_per_rank_padded(pl: Plan, stage: int) -> int:
    """Same, with the padded sizes the plan actually allocates."""
    K = pl.k_bytes
    if stage == 0:
        return (4 + K) * pl.psi_pad
    if stage == 1:
        return 4 * pl.psi_pad + K * pl.S
    if stage == 2:
        return 2 * pl.psi_pad + (2 + K) * pl.S
    if stage == 3:
        return (4 + K) * pl.S
    raise ValueError(stage)


# ---------------------------------------------------------- communication
def comm_elems_per_rank(pl: Plan) -> int:
    """Elements one rank sends per step under ring collectives."""
    one = (pl.nd - 1) * pl.S
    return 3 * one if pl.stage == 3 else 2 * one


def comm_bytes_per_rank(pl: Plan) -> int:
    return 2 * comm_elems_per_rank(pl)     # bf16 gradients and parameters


# ------------------------------------------------------------ HBM traffic
def hbm_step_bytes(pl: Plan, owner_view: bool = False,
                   with_reduced: bool = False) -> int:
    """Bytes the one-GPU step must move: read Nd bf16 gradient slices, read
    and write fp32 w, m, v, write the bf16 parameters (Nd replicas at stages
    0-2, the owner's shard at stage 3 or for a single-owner view), and
    optionally write the fp32 reduced gradient."""
    n = pl.S if owner_view else pl.psi_pad
    per = 2 * pl.nd + 24
    if owner_view or pl.stage == 3:
        per += 2
    else:
        per += 2 * pl.nd
    if with_reduced:
        per += 4
    return n * per


def hbm_guarded_step_bytes(pl: Plan, owner_view: bool = False) -> int:
    """The guarded step in two passes: the reduction reads the Nd bf16 rows
    and writes the fp32 sum; the update reads the sum and w, m, v and writes
    w, m, v and the parameters."""
    n = pl.S if owner_view else pl.psi_pad
    per = (2 * pl.nd + 4) + (4 + 24)
    per += 2 if (owner_view or pl.stage == 3) else 2 * pl.nd
    return n * per


def hbm_gather_bytes(pl: Plan, gathers_per_unit: int = 2) -> int:
    """Stage 3 materialisation: read 2 B and write 2 B per element of each
    unit, `gathers_per_unit` times per step (forward, then backward)."""
    return gathers_per_unit * sum(4 * n for n in pl.unit_len)


def storage_index(pl: Plan, cols):
    """Vector form of `locate`: logical indices -> rank-major storage index
    (owner * S + offset in the owner's block).  numpy int64 in and out."""
    import numpy as np
    cols = np.asarray(cols, dtype=np.int64)
    base = np.asarray(pl.unit_base, dtype=np.int64)
    u = np.searchsorted(base, cols, side="right") - 1
    j = cols - base[u]
    s = np.asarray(pl.unit_shard, dtype=np.int64)[u]
    owner = j // s
    off = np.asarray(pl.unit_offset, dtype=np.int64)[u] + (j - owner * s)
    return owner * pl.S + off


# ------------------------------------------------------ replicas, rank loss
def replicas(pl: Plan, what: str) -> int:
    """Ranks that hold a copy of each element's state, gradient or parameter.
    Concept page "ZeRO", table "三个阶段": ZeRO-1 shards the optimizer
    states (parameters and gradients stay replicated on every rank), ZeRO-2
    also the gradients, ZeRO-3 also the parameters; plain data parallelism
    (stage 0) replicates everything."""
    sharded_from = {"state": 1, "grad": 2, "param": 3}[what]
    return 1 if pl.stage >= sharded_from else pl.nd


def lost_rank_unrecoverable(pl: Plan, rank: int) -> int:
    """Real (unpadded) parameters whose optimizer state has no other copy once
    `rank` is lost: the ones it owns, unless the state is replicated."""
    if replicas(pl, "state") > 1:
        return 0
    n = 0
    for p in range(pl.psi_pad):
        u, owner, _, j = locate(pl, p)
        if owner == rank and j < pl.unit_len[u]:
            n += 1
    return n
