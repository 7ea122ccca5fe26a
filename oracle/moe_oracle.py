"""CPU oracle for one MoE layer: router -> top-k -> dispatch layout -> experts -> combine.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library (``dispatch_combine_grouped_b200``) and imports nothing from
it; the only common code is the seeded input generator in ``moe_inputs``.

Everything is float64 NumPy (inputs are converted exactly from their fp32/bf16 storage),
with no blocking, fusion or reordering beyond what each definition states.

Sources (web pages; cited by title and section):
  [EP-DeepEP]  "EP 解决的不是少算..." explainer, papers-3lj.pages.dev  .../explanations/ep_deepep
               §2 output equation y_t and tokens-per-expert n_e; §3 dispatch/combine as two
               all-to-alls with source-side bucketing by owner; §4 imbalance ratio;
               §6 the three index maps and the round-trip identity check.
  [DSMoE]      "深入浅出 DeepSeek MoE：EP 与 FSDP 经典二次开发实战指南", 0539edu.com
               "Expert Parallelism" section: the five-step naive MoE forward, the
               distributed transpose, and the combine's gate-weighted sum; VeOmni excerpt
               (preprocess / token_pre_all2all / tokens_post_all2all).
  [DeepEP]     "DeepEP" notes, lizn-zn.github.io, §2 the all-to-all transpose figure
               (block i->j of rank i lands as block i->j on rank j, source-major).
  [WideEP]     "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU", charlestar.github.io,
               sections "为什么要把 EP 做宽" (E_local, N_a), "一层里有两套并行布局"
               (attention-DP token shards), "Wide EP 的通信矩阵怎样扩张" (count matrix
               C_ij), "Group-limited routing 限制跨节点 fan-out", "三种负载必须同时平衡"
               (R_r = sum_i C_ir).
  [MoE-IV]     "MoE我们喜欢你（四）：DeepEP 与 GroupedGEMM 如何拆解通信和计算瓶颈",
               §4 pipeline permute -> a2a -> grouped_gemm -> a2a -> unpermute_and_weighted_sum.

Readings where the pages are silent (each is listed in the design notes):
  * SwiGLU: Expert_e(x) = W_down (SiLU(W_gate x) * (W_up x)), SiLU(z) = z / (1 + e^-z);
    W13 rows [0, I) are the gate projection and rows [I, 2I) the up projection.
  * Selection is made on the router logit (softmax and sigmoid are strictly monotone);
    ties go to the lower expert (or group) index; slot order is descending key.
  * Group score = max key inside the group.
  * Source rank of token t = t // ceil(N / P) (contiguous attention-DP shards).
  * Send buffer order = (source, owner, assignment index a = t*k + slot).
  * Owner j's receive buffer is source-major; inside it, a stable sort by expert id
    gives the expert-local order; owners' buffers follow each other in owner order.
  * Return row = send slot (the combine all-to-all is the inverse transpose).
  * Shared experts are added with weight 1.
  * A correction bias (bias_mode "selection") shifts the selection keys only.
  * Capacity ([EP-DeepEP] §4, capacity factor): an expert receives at most
    ceil(factor * N * k / E) assignments, the first ones in ascending a; the others are
    dropped (id -1): they take no row and add nothing to y, and the gates of the kept
    assignments are left as they are.
"""
from __future__ import annotations

import itertools

import numpy as np

TILE_M = 128  # row-block size used by the tile prefix (tile_off) in the layout contract


def f64(a) -> np.ndarray:
    """Exact conversion of a NumPy array or CPU/GPU torch tensor to float64 NumPy."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def i64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").long().numpy()
    return np.asarray(a, dtype=np.int64)


# ---------------------------------------------------------------------------------------
# Step 1 — gate (router) logits.  [DSMoE] naive forward, step 1; [EP-DeepEP] §2 "z in R^{NxE}".
# ---------------------------------------------------------------------------------------
def router_logits(x, w_gate, bias=None) -> np.ndarray:
    """z[t, e] = <x_t, W_g[e]> (+ b_e), in float64.  w_gate is stored [E, d]."""
    z = f64(x) @ f64(w_gate).T
    if bias is not None:
        z = z + f64(bias)[None, :]
    return z


# ---------------------------------------------------------------------------------------
# Step 2 — expert selection I_t.  [DSMoE] step 2; [WideEP] group-limited routing.
# ---------------------------------------------------------------------------------------
def _descending_stable(keys_row: np.ndarray) -> np.ndarray:
    # order by descending key; equal keys keep ascending index (lower index first)
    return np.argsort(-keys_row, kind="stable")


def select_experts(keys, k: int, n_groups: int = 1, topk_groups: int = 1) -> np.ndarray:
    """Top-k expert ids per token, slot 0 = largest key, ties to the lower index.

    With n_groups > 1 the E experts form n_groups contiguous groups; a token first keeps
    the topk_groups groups with the largest group score (max key in the group, ties to
    the lower group index), then takes its top-k among the experts of those groups.
    ``keys`` may be float64 logits or the float32 logits of another implementation
    (comparisons are exact either way).
    """
    keys = np.asarray(keys)
    N, E = keys.shape
    ids = np.empty((N, k), dtype=np.int64)
    gsize = E // n_groups
    for t in range(N):
        row = keys[t].astype(np.float64)
        if n_groups > 1:
            gscore = row.reshape(n_groups, gsize).max(axis=1)
            kept = _descending_stable(gscore)[:topk_groups]
            allowed = np.zeros(E, dtype=bool)
            for g in kept:
                allowed[g * gsize:(g + 1) * gsize] = True
            cand = np.flatnonzero(allowed)              # ascending expert ids
            order = cand[_descending_stable(row[cand])]
        else:
            order = _descending_stable(row)
        ids[t] = order[:k]
    return ids


def brute_force_select(keys, k: int, n_groups: int = 1, topk_groups: int = 1) -> np.ndarray:
    """Independent selection by enumeration (tiny E only).

    The chosen group set is the lexicographically first (in ascending group ids) among
    the sets whose sorted group-score multiset is largest; the chosen expert set is the
    lexicographically first k-subset of the allowed experts maximising the sorted key
    multiset.  Slots are then ordered by descending key, ties by ascending index.
    """
    keys = np.asarray(keys, dtype=np.float64)
    N, E = keys.shape
    gsize = E // n_groups
    out = np.empty((N, k), dtype=np.int64)
    for t in range(N):
        row = keys[t]
        allowed = list(range(E))
        if n_groups > 1:
            gscore = [max(row[g * gsize:(g + 1) * gsize]) for g in range(n_groups)]
            best = None
            for gs in itertools.combinations(range(n_groups), topk_groups):
                val = sorted((gscore[g] for g in gs), reverse=True)
                # larger multiset wins; among equal multisets the earlier (lexicographic)
                # combination wins, which prefers lower group ids on ties
                if best is None or val > best[0]:
                    best = (val, gs)
            allowed = [e for g in best[1] for e in range(g * gsize, (g + 1) * gsize)]
        best = None
        for sub in itertools.combinations(allowed, k):
            val = sorted((row[e] for e in sub), reverse=True)
            if best is None or val > best[0]:
                best = (val, sub)
        chosen = sorted(best[1], key=lambda e: (-row[e], e))
        out[t] = chosen
    return out


# ---------------------------------------------------------------------------------------
# Step 3 — gate weights g_{t,e}.  [EP-DeepEP] §2; renormalisation as named in [MoE-IV] §4.2.
# ---------------------------------------------------------------------------------------
def gate_weights(logits, ids, score: str = "softmax", renormalize: bool = True) -> np.ndarray:
    z = f64(logits)
    ids = i64(ids)
    N, k = ids.shape
    chosen = np.take_along_axis(z, ids, axis=1)
    if score == "softmax":
        if renormalize:
            m = chosen.max(axis=1, keepdims=True)
            num = np.exp(chosen - m)
            return num / num.sum(axis=1, keepdims=True)
        m = z.max(axis=1, keepdims=True)
        den = np.exp(z - m).sum(axis=1, keepdims=True)
        return np.exp(chosen - m) / den
    if score == "sigmoid":
        s = 1.0 / (1.0 + np.exp(-chosen))
        if renormalize:
            return s / s.sum(axis=1, keepdims=True)
        return s
    raise ValueError(score)


def gate_logits(cfg, x, w_gate, bias):
    """Logits the gate weights are computed from: x W_g^T + b, or with a correction bias
    (bias_mode "selection", named as router correction_bias in [MoE-IV] §4.2) the
    unbiased x W_g^T — the bias then only steers which experts are selected."""
    if getattr(cfg, "bias_mode", "logits") == "selection":
        return router_logits(x, w_gate, None)
    return router_logits(x, w_gate, bias)


# ---------------------------------------------------------------------------------------
# Step 4 — dispatch layout.  [EP-DeepEP] §2 (n_e), §3 (bucket by owner at the source),
# §6 (three maps); [WideEP] C_ij and R_r; [DeepEP] §2 transpose; [DSMoE] VeOmni excerpt.
# ---------------------------------------------------------------------------------------
def default_owner(E: int, P: int) -> np.ndarray:
    """Contiguous placement: owner j holds experts [j*E/P, (j+1)*E/P)  ([WideEP] E_local)."""
    if E % P != 0:
        raise ValueError("contiguous placement needs E % P == 0")
    return np.arange(E, dtype=np.int64) // (E // P)


def source_of_token(N: int, P: int) -> np.ndarray:
    """Attention-DP shards: source rank i holds tokens [i*ceil(N/P), (i+1)*ceil(N/P))."""
    shard = -(-N // P)
    return np.arange(N, dtype=np.int64) // shard


def dispatch_layout(ids, E: int, P: int, expert_owner=None, S: int = 0) -> dict:
    """All layout metadata of the dispatch, from the definitions.

    Returns int64 arrays:
      n_e[E], expert_off[E+1], C[P,P], send_off[P,P], recv_off[P+1],
      tok2send[A], send2row[A], ret2tok[A], tok2row[A], row2tok[A], tile_off[E+S+1].
    Dropped assignments (id -1) take no row and no send slot: their tok2send / tok2row
    are -1, and the slots / rows past the A_kept used ones are -1 in send2row, ret2tok
    and row2tok; expert_off[E] = A_kept.
    """
    ids = i64(ids)
    N, k = ids.shape
    A = N * k
    owner = default_owner(E, P) if expert_owner is None else i64(expert_owner)
    flat_all = ids.reshape(-1)                   # expert of assignment a = t*k + slot
    kept = np.flatnonzero(flat_all >= 0)         # assignments that are dispatched
    A_kept = len(kept)
    flat = flat_all[kept]
    src = source_of_token(N, P)[kept // k]       # source rank of each kept assignment
    dst = owner[flat]                            # destination owner of each kept assignment

    n_e = np.bincount(flat, minlength=E).astype(np.int64)

    C = np.zeros((P, P), dtype=np.int64)
    for i, j in zip(src, dst):
        C[i, j] += 1

    # Send buffer: each source buckets its assignments by owner, keeping token order.
    order_send = np.lexsort((kept, dst, src))    # primary src, then owner, then a
    send_list = kept[order_send]                 # assignment in each send slot
    tok2send = np.full(A, -1, dtype=np.int64)
    tok2send[send_list] = np.arange(A_kept)
    send_off = np.zeros((P, P), dtype=np.int64)
    flatC = C.reshape(-1)
    send_off.reshape(-1)[1:] = np.cumsum(flatC)[:-1]

    # Receive buffers (the transpose): owner j gets blocks i->j for i = 0..P-1 in order.
    rows = []
    R = np.zeros(P, dtype=np.int64)
    dst_of = np.full(A, -1, dtype=np.int64)
    dst_of[kept] = dst
    for j in range(P):
        recv_j = send_list[dst_of[send_list] == j]  # source-major, token order inside
        R[j] = len(recv_j)
        order = np.argsort(flat_all[recv_j], kind="stable")   # expert-local order
        rows.append(recv_j[order])
    row_list = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    recv_off = np.zeros(P + 1, dtype=np.int64)
    recv_off[1:] = np.cumsum(R)

    tail = np.full(A - A_kept, -1, dtype=np.int64)
    row2tok = np.concatenate([row_list, tail])
    tok2row = np.full(A, -1, dtype=np.int64)
    tok2row[row_list] = np.arange(A_kept)
    send2row = np.concatenate([tok2row[send_list], tail])
    ret2tok = np.concatenate([send_list, tail])

    # expert_off[e]: first row of expert e; experts follow owner order, then id order.
    expert_off = np.zeros(E + 1, dtype=np.int64)
    run = 0
    for j in range(P):
        for e in range(E):
            if owner[e] == j:
                expert_off[e] = run
                run += n_e[e]
    expert_off[E] = A_kept

    # Row-block prefix over groups in id order (routed experts, then S shared groups of N rows).
    blocks = [-(-int(n) // TILE_M) for n in n_e] + [-(-N // TILE_M)] * S
    tile_off = np.zeros(E + S + 1, dtype=np.int64)
    tile_off[1:] = np.cumsum(blocks)

    return dict(n_e=n_e, expert_off=expert_off, C=C, send_off=send_off, recv_off=recv_off,
                tok2send=tok2send, send2row=send2row, ret2tok=ret2tok, tok2row=tok2row,
                row2tok=row2tok, tile_off=tile_off)


def _ep_receive_lists(flats, owner, E: int, P: int) -> list:
    """Owner j's receive rows as (source i, local a): the experts j owns in ascending id,
    each expert's assignments from source 0, then source 1, ..., each source's in ascending
    local index a ([DeepEP] §2: blocks arrive in source order; the expert-local order is
    ascending (t, slot))."""
    recv = [[] for _ in range(P)]
    for e in range(E):
        j = int(owner[e])
        for i, f in enumerate(flats):
            for a in np.flatnonzero(f == e):
                recv[j].append((i, int(a)))
    return recv


def ep_layout(ids_per_rank, E: int, P: int, expert_owner=None, capacity=None) -> dict:
    """The dispatch across P ranks, each rank one source of tokens and the owner of some
    experts ([EP-DeepEP] §3: tokens go to the owner of their expert and come back to
    their source; [DeepEP] §2: owner j receives the blocks from sources 0, 1, ... in
    order; [WideEP] the count matrix).  ids_per_rank[i] is rank i's [n_i, k] top-k ids
    (n_i may differ, -1 = dropped).

    Owner j's receive rows, from the definition: for each expert e that j owns, in
    ascending id, the assignments to e of source 0, then of source 1, ..., each source's
    in ascending local index a = t*k + slot.  With `capacity`, rows at or past it are not
    received.  Returns
      cnt[P, E]          counts of each source (the rows exchanged first)
      recv[j]            [R_j, 2] array of (source i, local a) per receive row of owner j
      R[P]               rows each owner is sent (before the capacity)
      dest[i]            [n_i*k]: owner * capacity + row, -1 for dropped / not received
      owned[j]           experts owner j holds, ascending
      owner_n_e[j], owner_off[j]  rows received per owned expert and their first row
                         (capped at capacity; owner_off[j][-1] = rows received)
    """
    owner = default_owner(E, P) if expert_owner is None else i64(expert_owner)
    flats = [i64(x).reshape(-1) for x in ids_per_rank]
    cnt = np.zeros((P, E), dtype=np.int64)
    for i, f in enumerate(flats):
        kept = f[f >= 0]
        cnt[i] = np.bincount(kept, minlength=E)[:E]
    recv = _ep_receive_lists(flats, owner, E, P)
    R = np.array([len(r) for r in recv], dtype=np.int64)
    cap = int(capacity) if capacity is not None else max(int(R.max()), 1)
    dest = [np.full(len(f), -1, dtype=np.int64) for f in flats]
    for j in range(P):
        for row, (i, a) in enumerate(recv[j]):
            if row < cap:
                dest[i][a] = j * cap + row
    n_tot = cnt.sum(axis=0)
    owned, owner_n_e, owner_off = [], [], []
    for j in range(P):
        mine = [e for e in range(E) if owner[e] == j]
        first, rows, run = [], [], 0
        for e in mine:
            f0 = min(run, cap)
            first.append(f0)
            rows.append(min(int(n_tot[e]), cap - f0))
            run += int(n_tot[e])
        owned.append(np.array(mine, dtype=np.int64))
        owner_n_e.append(np.array(rows, dtype=np.int64))
        owner_off.append(np.array(first + [min(run, cap)], dtype=np.int64))
    return dict(cnt=cnt, recv=[np.array(r, dtype=np.int64).reshape(-1, 2) for r in recv], R=R, dest=dest,
                capacity=cap, owned=owned, owner_n_e=owner_n_e, owner_off=owner_off)


def imbalance(counts) -> float:
    """max / mean of a load vector ([EP-DeepEP] §4)."""
    c = np.asarray(counts, dtype=np.float64)
    return float(c.max() / c.mean())


# ---------------------------------------------------------------------------------------
# Steps 3'-5 — token movement and experts.  [MoE-IV] §4: permute, grouped FFN, unpermute
# with the weighted sum.  [DSMoE] steps 3-5.
# ---------------------------------------------------------------------------------------
def silu(z):
    return z / (1.0 + np.exp(-z))


def swiglu_expert(x_rows, w13_e, w2_e) -> np.ndarray:
    """Expert_e(x) = W_down (SiLU(W_gate x) * (W_up x)) for a block of rows, float64."""
    x_rows = f64(x_rows)
    w13_e = f64(w13_e)
    I = w13_e.shape[0] // 2
    gate = x_rows @ w13_e[:I].T
    up = x_rows @ w13_e[I:].T
    return (silu(gate) * up) @ f64(w2_e).T


def permute(x, layout, k: int) -> np.ndarray:
    """x_perm[tok2row[a]] = x[a // k]  (token rows in expert-contiguous order); rows past
    the kept ones stay zero."""
    x = f64(x)
    tok2row = layout["tok2row"]
    out = np.zeros((len(tok2row), x.shape[1]))
    a = np.flatnonzero(tok2row >= 0)
    out[tok2row[a]] = x[a // k]
    return out


def combine(o_rows, layout, gates, N: int, k: int, shared_out=None) -> np.ndarray:
    """y_t = sum_slot g_{t,slot} * o[tok2row[t*k+slot]]  (+ sum of shared expert outputs)."""
    o_rows = f64(o_rows)
    g = f64(gates)
    y = np.zeros((N, o_rows.shape[1]))
    for slot in range(k):
        rows = layout["tok2row"][np.arange(N) * k + slot]
        live = rows >= 0  # a dropped assignment adds nothing
        y[live] += g[live, slot:slot + 1] * o_rows[rows[live]]
    if shared_out is not None:
        for so in shared_out:
            y += so
    return y


def experts_on_rows(x_perm, layout, w13, w2, E: int) -> np.ndarray:
    """Run Expert_e on its contiguous rows [expert_off[e], expert_off[e]+n_e)."""
    out = np.zeros((x_perm.shape[0], f64(w2[0]).shape[0]))
    for e in range(E):
        n = layout["n_e"][e]
        if n == 0:
            continue
        r0 = layout["expert_off"][e]
        out[r0:r0 + n] = swiglu_expert(x_perm[r0:r0 + n], w13[e], w2[e])
    return out


def moe_layer(cfg, x, w_gate, bias, w13, w2, expert_owner=None, select_keys=None) -> dict:
    """The whole layer in the pages' order (gate, select, dispatch, experts, combine).

    ``select_keys`` optionally replaces the logits used for selection (e.g. another
    implementation's fp32 logits); the gate values always come from the float64 logits.
    """
    z = router_logits(x, w_gate, bias)
    keys = z if select_keys is None else np.asarray(select_keys)
    ids = select_experts(keys, cfg.k, cfg.n_groups, cfg.topk_groups)
    g = gate_weights(gate_logits(cfg, x, w_gate, bias), ids, cfg.score, cfg.renormalize)
    lay = dispatch_layout(ids, cfg.E, cfg.P, expert_owner, cfg.S)
    xp = permute(x, lay, cfg.k)
    o = experts_on_rows(xp, lay, w13, w2, cfg.E)
    shared = [swiglu_expert(x, w13[cfg.E + s], w2[cfg.E + s]) for s in range(cfg.S)]
    y = combine(o, lay, g, cfg.N, cfg.k, shared)
    return dict(logits=z, ids=ids, gates=g, layout=lay, y=y)


def moe_tokens_direct(cfg, x, ids, gates, w13, w2, tokens) -> np.ndarray:
    """y_t straight from the output equation for selected tokens (no layout):
    y_t = sum_{e in I_t} g_{t,e} Expert_e(x_t) + sum_s Shared_s(x_t)   ([EP-DeepEP] §2)."""
    x = f64(x)
    ids = i64(ids)
    g = f64(gates)
    tokens = np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(tokens), x.shape[1]))
    by_expert = {}
    for n, t in enumerate(tokens):
        for slot in range(ids.shape[1]):
            if ids[t, slot] >= 0:  # a dropped assignment adds nothing
                by_expert.setdefault(int(ids[t, slot]), []).append((n, t, slot))
    for e, lst in sorted(by_expert.items()):
        rows = np.array([t for _, t, _ in lst])
        oe = swiglu_expert(x[rows], w13[e], w2[e])
        for (n, t, slot), o in zip(lst, oe):
            out[n] += g[t, slot] * o
    for s in range(cfg.S):
        out += swiglu_expert(x[tokens], w13[cfg.E + s], w2[cfg.E + s])
    return out


def capacity(factor: float, N: int, k: int, E: int) -> int:
    """Assignments one expert may receive: ceil(factor * N * k / E) ([EP-DeepEP] §4: the
    uniform share N k / E times the capacity factor)."""
    return int(np.ceil(factor * N * k / E))


def capacity_keep(ids, E: int, cap: int) -> np.ndarray:
    """Ids with every assignment past the first `cap` of its expert (ascending a) set to -1."""
    ids = i64(ids)
    flat = ids.reshape(-1).copy()
    for e in range(E):
        rows = np.flatnonzero(flat == e)
        flat[rows[cap:]] = -1
    return flat.reshape(ids.shape)

