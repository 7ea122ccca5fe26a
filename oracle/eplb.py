"""CPU oracle for redundant expert slots (EPLB): plan, assignment to replicas, weights.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library and imports nothing from it.

Source: "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU" (charlestar.github.io):
  * "为什么要把 EP 做宽": E logical routed experts plus R redundant copies give E + R
    physical experts, E_local = (E + R) / P_e per owner rank.
  * "DeepSeek-V3/R1 的两个具体布局": 256 + 32 = 288 physical slots, 9 per rank at EP32.
  * "Expert 副本在 Wide EP 中还有整除作用": replicas copy hot experts and make the slot
    count divisible by the EP width; a logical expert's assignments are spread over its
    replicas; which experts to copy follows the measured workload.
  * "三种负载必须同时平衡": the expert-parallel balancer minimises the largest expert /
    receive load, R_r = sum_i C_ir.
  * "Group-limited routing": the router's choice is model semantics; only the replica of
    the chosen logical expert may be picked by the runtime.

The pages fix what the plan is for, not an algorithm.  Readings taken here (each listed
in the design notes), in the plainest form that meets the stated goal:
  1. Replica counts: every logical expert keeps one copy; each of the R extra copies in
     turn goes to the expert with the largest load per copy, load_e / r_e (ties to the
     lower expert id).  Giving the next copy to the current maximum is what lowers the
     maximum, so this minimises max_e load_e / r_e.
  2. Placement: copy c of expert e carries the rows reading 4 gives it,
     floor(load_e / r_e) + (1 if c < load_e mod r_e else 0).  The E + R copies are taken
     in descending load order (ties: lower expert id, then lower copy number) and each
     goes to the owner with free room (E_local slots per owner) that holds no copy of the
     same expert yet if there is one, then the smallest load so far, then the lower owner.
  3. Slot ids: owner j holds slots [j E_local, (j+1) E_local), in ascending (expert id,
     copy number) order; a logical expert's replicas are listed by copy number.
  4. Assignment: the q-th assignment of logical expert e in ascending a = t k + slot order
     goes to replica q mod r_e, so the copies of e share its n_e to within one row.
"""
from __future__ import annotations

import numpy as np


def replica_counts(load, R: int) -> np.ndarray:
    """Reading 1: copies per logical expert, sum = E + R."""
    load = np.asarray(load, dtype=np.int64)
    r = np.ones(len(load), dtype=np.int64)
    for _ in range(R):
        best = 0
        for e in range(1, len(load)):
            # load[e] / r[e] > load[best] / r[best], exact in integers
            if load[e] * r[best] > load[best] * r[e]:
                best = e
        r[best] += 1
    return r


def copy_load(load_e: int, r_e: int, c: int) -> int:
    """Rows copy c of an expert with load_e rows and r_e copies receives (reading 4)."""
    return load_e // r_e + (1 if c < load_e % r_e else 0)


def plan(load, R: int, P: int) -> dict:
    """Readings 1-3.  Returns copies [E], replica_off [E+1], replica_slots [E+R] (slot of
    copy c of expert e at replica_off[e] + c), slot_expert [E+R], slot_owner [E+R]."""
    load = np.asarray(load, dtype=np.int64)
    E = len(load)
    S = E + R
    if S % P != 0:
        raise ValueError("E + R must be a multiple of P")
    per = S // P
    r = replica_counts(load, R)
    copies = [(copy_load(int(load[e]), int(r[e]), c), e, c) for e in range(E) for c in range(r[e])]
    # descending load, then ascending expert id, then ascending copy number
    order = sorted(copies, key=lambda u: (-u[0], u[1], u[2]))

    owner_load = [0] * P
    owner_room = [per] * P
    holds = [set() for _ in range(P)]
    owner_of = {}
    for (cl, e, c) in order:
        best = -1
        for j in range(P):
            if owner_room[j] == 0:
                continue
            if best < 0:
                best = j
                continue
            fresh_j, fresh_b = e not in holds[j], e not in holds[best]
            if fresh_j != fresh_b:
                if fresh_j:
                    best = j
                continue
            if owner_load[j] < owner_load[best]:
                best = j
        owner_of[(e, c)] = best
        owner_load[best] += cl
        owner_room[best] -= 1
        holds[best].add(e)

    slot_expert = np.empty(S, dtype=np.int64)
    slot_owner = np.empty(S, dtype=np.int64)
    replica_off = np.zeros(E + 1, dtype=np.int64)
    replica_off[1:] = np.cumsum(r)
    replica_slots = np.empty(S, dtype=np.int64)
    for j in range(P):
        mine = sorted((e, c) for (e, c), o in owner_of.items() if o == j)
        for i, (e, c) in enumerate(mine):
            slot = j * per + i
            slot_expert[slot] = e
            slot_owner[slot] = j
            replica_slots[replica_off[e] + c] = slot
    return {"replica_off": replica_off, "replica_slots": replica_slots,
            "slot_expert": slot_expert, "slot_owner": slot_owner, "copies": r,
            "owner_load": np.asarray(owner_load, dtype=np.int64)}


def assign(ids, replica_off, replica_slots) -> np.ndarray:
    """Reading 4: physical slot of every assignment, same shape as ids."""
    ids = np.asarray(ids, dtype=np.int64)
    flat = ids.reshape(-1)
    replica_off = np.asarray(replica_off, dtype=np.int64)
    replica_slots = np.asarray(replica_slots, dtype=np.int64)
    out = np.empty_like(flat)
    for e in range(len(replica_off) - 1):
        rows = np.flatnonzero(flat == e)  # ascending a
        r = replica_off[e + 1] - replica_off[e]
        q = np.arange(len(rows))
        out[rows] = replica_slots[replica_off[e] + q % r]
    return out.reshape(ids.shape)


def physical_weights(w, slot_expert, E: int):
    """Weights of the physical slots (a copy of each slot's logical expert), followed by
    the shared experts (indices E.. of the logical array) unchanged.  ``w`` is a torch
    tensor [E+S, ...] on any device; plain indexing, no arithmetic."""
    import torch
    idx = torch.as_tensor(np.asarray(slot_expert, dtype=np.int64), device=w.device)
    return torch.cat([w.index_select(0, idx), w[E:]], dim=0)
