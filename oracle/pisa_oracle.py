"""Plain CPU oracle of PISA pyramid block-sparse attention (numpy, fp32; fp64 brute force).

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg do. It shares no code with the CUDA library.

What it follows (the pages give no equations, pseudo-code or constants; each
open point takes the plainest reading, listed as R1..R18 in the design notes):

* "Attention clairsemee PISA : noyaux Triton sans matrice de scores"
  (irisproject.cloud), sections "Une pyramide de cles plutot qu'un tapis
  uniforme" and "Le pooling comme premiere reduction": keys are grouped into
  small packets, then packets of packets, each level summarising the one
  below by pooling  ->  ``build_pyramid``.
* same page, section "La selection top-K guidee par la pyramide": the K most
  relevant blocks are chosen by descending the levels, pruning hard at the
  top and refining below  ->  ``select_blocks``.
* same page, section "Des noyaux Triton qui ne materialisent rien": similarity,
  selection and aggregation computed without writing the N x N score matrix;
  the oracle may write it (it is the slow reference)  ->  ``attend``.
* "L'Attention Lineaire : Comment l'IA Accelere ses Calculs..." (techfacile.cc),
  section "Le Probleme du Cout Quadratique de l'Attention Classique": dense
  softmax attention, QK^T -> softmax -> V  ->  ``dense_attention`` (fp64).
* "Dropping the Anchor ... via Pulsar Attention" (gist.science), section
  "Phase 2 : Encodage de la requete globale": partial attentions over disjoint
  key sets are combined by an online-softmax merge  ->  ``merge_partials``.
* PISA page, section "La selection top-K guidee par la pyramide" (top-K variants
  may be tuned per domain) and the Pulsar page's fixed attention-sink prefix:
  blocks that are always kept (sink, local)  ->  ``forced_set`` and the
  ``forced`` argument of ``select_blocks``.
* PISA page, section "Des noyaux Triton qui ne materialisent rien" (the memory
  footprint stays stable as the context grows): a pyramid over a KV cache with
  spare capacity, every node the mean of the keys it covers among the valid
  rows  ->  ``build_pyramid_capacity``.
* PISA page, section "Ce que cela change pour vous" (for those who train as well
  as deploy models) and the key points' "training as well as inference":
  gradients of the attention step through a fixed selection  ->
  ``attend_backward``, ``backward``.

Parity pins (tests/test_oracle_pins.py) tie every function here to a closed
form, a brute-force computation or an invariant; none is "parity unpinned".
"""
from __future__ import annotations

import itertools
import math

import numpy as np

F32 = np.float32
NEAR_TIE_REL = 1e-3     # near-tie: relative score margin at a pruning level below this


# ----------------------------------------------------------------------------- pyramid

def level_sizes(n0: int, factor: int) -> list[int]:
    """Node count of every pyramid level: n_{l+1} = ceil(n_l / f), built while n_l > f (R1)."""
    sizes = [n0]
    while sizes[-1] > factor:
        sizes.append(-(-sizes[-1] // factor))
    return sizes


def node_span(n0: int, factor: int, level: int, c: int) -> tuple[int, int]:
    """First and last level-0 block covered by node c of a level."""
    width = factor ** level
    return c * width, min((c + 1) * width, n0) - 1


def children(n_below: int, factor: int, c: int) -> list[int]:
    """Children of node c in the level below (the last node of a level may have fewer than f)."""
    return list(range(c * factor, min(c * factor + factor, n_below)))


def block_means(k_plane: np.ndarray, block: int) -> np.ndarray:
    """Level 0: the fp32 mean of the `block` keys of every key block. k_plane [N, D] -> [N/block, D]."""
    n0 = k_plane.shape[0] // block
    blocks = k_plane[:n0 * block].astype(F32).reshape(n0, block, -1)
    return blocks.sum(axis=1, dtype=F32) / F32(block)


def build_pyramid(k_plane: np.ndarray, block: int, factor: int) -> list[np.ndarray]:
    """Key pyramid of one (batch, KV head) plane: list of levels, level l is [n_l, D] fp32.

    Level 0 holds the key-block means. A node of level l+1 is the mean of its
    children weighted by how many level-0 blocks each covers (R2); for a node
    whose f children are all full this is the plain mean of the children, and
    in every case it equals the mean of all the keys the node covers.
    """
    levels = [block_means(k_plane, block)]
    n0 = levels[0].shape[0]
    sizes = level_sizes(n0, factor)
    for l in range(1, len(sizes)):
        below = levels[l - 1]
        cur = np.zeros((sizes[l], below.shape[1]), dtype=F32)
        for c in range(sizes[l]):
            acc = np.zeros(below.shape[1], dtype=F32)
            total = 0
            for ch in children(sizes[l - 1], factor, c):
                lo, hi = node_span(n0, factor, l - 1, ch)
                cnt = hi - lo + 1
                acc += F32(cnt) * below[ch]
                total += cnt
            cur[c] = acc / F32(total)
        levels.append(cur)
    return levels


def build_pyramid_capacity(k_plane: np.ndarray, block: int, factor: int, kv_len: int) -> list[np.ndarray]:
    """Key pyramid of a KV cache with spare capacity (R17): k_plane [capacity, D] of which the
    first kv_len rows hold keys. The levels have the sizes of the whole capacity; every node is
    the mean of the keys it covers among the first kv_len (weights count only those blocks), and
    a node over none of them is 0. With kv_len = capacity this is ``build_pyramid``.
    """
    n0_cap = k_plane.shape[0] // block
    nv = kv_len // block
    d = k_plane.shape[1]
    sizes = level_sizes(n0_cap, factor)
    lev0 = np.zeros((n0_cap, d), dtype=F32)
    if nv > 0:
        lev0[:nv] = block_means(k_plane[:nv * block], block)
    levels = [lev0]
    for l in range(1, len(sizes)):
        below = levels[l - 1]
        cur = np.zeros((sizes[l], d), dtype=F32)
        for c in range(sizes[l]):
            acc = np.zeros(d, dtype=F32)
            total = 0
            for ch in children(sizes[l - 1], factor, c):
                lo, hi = node_span(n0_cap, factor, l - 1, ch)
                cnt = max(0, min(hi, nv - 1) - lo + 1)
                if cnt == 0:
                    continue
                acc += F32(cnt) * below[ch]
                total += cnt
            if total > 0:
                cur[c] = acc / F32(total)
        levels.append(cur)
    return levels


# ----------------------------------------------------------------------------- query summary

def query_summary(q_heads: np.ndarray, rows_per_block: int) -> np.ndarray:
    """Mean query of every query block over the heads that share one selection (R3, R4).

    q_heads [g, Nq, D] -> [Nq / rows_per_block, D] fp32. Group-shared selection
    passes the g query heads of a KV head; per-query-head selection passes one
    head; decode passes rows_per_block = 1 (the single query token).
    """
    g, nq, d = q_heads.shape
    nqb = nq // rows_per_block
    x = q_heads[:, :nqb * rows_per_block].astype(F32).reshape(g, nqb, rows_per_block, d)
    return x.sum(axis=(0, 2), dtype=F32) / F32(g * rows_per_block)


# ----------------------------------------------------------------------------- selection

def node_value(levels: list[np.ndarray], factor: int, level: int, c: int, last: int) -> np.ndarray:
    """Summary vector a query block scores node c against.

    `last` is the last level-0 block the query block may use (causal: its own
    index). A node wholly at or before `last` uses its pyramid value. The node
    that straddles `last` is summarised by the mean of its eligible level-0
    block means only, so no future key enters the selection (R6).
    """
    n0 = levels[0].shape[0]
    lo, hi = node_span(n0, factor, level, c)
    if hi <= last:
        return levels[level][c]
    return levels[0][lo:last + 1].sum(axis=0, dtype=F32) / F32(last + 1 - lo)


def score(qbar: np.ndarray, node: np.ndarray) -> F32:
    """Relevance of a node: the raw fp32 dot product q_bar . node (R5)."""
    return F32(np.dot(qbar.astype(F32), node.astype(F32)))


def rank_key(score_value: float, node: int) -> tuple[float, int]:
    """Sort key of a candidate: higher score first, then lower node index (R8)."""
    return (-float(score_value), node)


def forced_set(forced: int, local: int, topk: int) -> list[int]:
    """Blocks a selection variant always keeps (R16): key block 0 (attention sink, bit 1) and the
    query's own block `local` (bit 2), without repeats, at most K of them, the sink first."""
    out: list[int] = []
    if forced & 1:
        out.append(0)
    if forced & 2 and local not in out:
        out.append(local)
    return out[:topk]


def select_blocks(qbar: np.ndarray, levels: list[np.ndarray], factor: int, topk: int,
                  last: int, budgets: list[int] | None = None, forced: list[int] | None = None) -> dict:
    """Descend the pyramid for one query summary and keep the top-K key blocks.

    Start with every eligible node of the top level; at each level score the
    candidates, keep the best K_l (all of them when there are no more than
    K_l), and pass the eligible children of the kept nodes down (R9: K_l = K by
    default). Returns the kept level-0 blocks sorted ascending (R12), the
    smallest relative margin s_(K) - s_(K+1) met at a pruning level (R10), and
    the number of candidates scored (work bound, O(N log N)).

    `forced` (R16) lists level-0 blocks that are always kept: they are taken out
    of the level-0 candidates, whose budget drops by their number, and added to
    the result. Coarser levels are unchanged.
    """
    n_levels = len(levels)
    n0 = levels[0].shape[0]
    if budgets is None:
        budgets = [topk] * n_levels
    top = n_levels - 1
    cands = [c for c in range(levels[top].shape[0]) if node_span(n0, factor, top, c)[0] <= last]
    margin = math.inf
    n_scored = 0
    kept: list[int] = []
    forced = [] if forced is None else list(forced)
    for l in range(top, -1, -1):
        if l == 0 and forced:
            cands = [c for c in cands if c not in forced]
        scores = [score(qbar, node_value(levels, factor, l, c, last)) for c in cands]
        n_scored += len(cands)
        order = sorted(range(len(cands)), key=lambda t: rank_key(scores[t], cands[t]))
        k_l = budgets[l] - (len(forced) if l == 0 else 0)
        if k_l == 0:
            kept = []
        elif len(cands) > k_l:
            s_k, s_k1 = float(scores[order[k_l - 1]]), float(scores[order[k_l]])
            rel = (s_k - s_k1) / max(abs(s_k), abs(s_k1), 1e-30)
            margin = min(margin, rel)
            kept = [cands[t] for t in order[:k_l]]
        else:
            kept = list(cands)
        if l > 0:
            n_below = levels[l - 1].shape[0]
            cands = sorted(ch for c in kept for ch in children(n_below, factor, c)
                           if node_span(n0, factor, l - 1, ch)[0] <= last)
    return {"idx": sorted(kept + forced), "margin": margin, "n_scored": n_scored}


def _near(a: float, b: float, rel_tol: float) -> bool:
    """Two scores within the near-tie tolerance of each other (R10's relative measure)."""
    return abs(a - b) <= rel_tol * max(abs(a), abs(b), 1e-30)


def selection_is_admissible(qbar: np.ndarray, levels: list[np.ndarray], factor: int, topk: int, last: int,
                            row, budgets: list[int] | None = None, forced: list[int] | None = None,
                            rel_tol: float = NEAR_TIE_REL, max_branches: int = 4096) -> tuple[bool, str]:
    """Whether a selection row computed elsewhere is one the descent of ``select_blocks`` can reach
    when every near-tie at a pruning level may be resolved either way (R10).

    ``row`` lists kept level-0 blocks in ascending order, then -1 padding (R12). It must be well
    formed: no entry after the padding, strictly ascending (so distinct), every block eligible
    (0 <= j <= last) and every forced block present (R16). Then the descent is replayed with this
    oracle's fp32 scores: at a pruning level whose K_l-th and (K_l+1)-th scores are within
    ``rel_tol`` of each other (a near-tie), the candidates whose scores lie within ``rel_tol`` of
    either form a band, those above the band are kept, those below it dropped, and any choice of
    band members that fills the budget is one branch; a level without a near-tie keeps its top
    K_l. With ``rel_tol = 0`` the branches are exactly the ways of breaking equal scores. The row is
    admissible if some branch ends with exactly its blocks. Branches are pruned by the row itself:
    every ancestor j // f^l of a row block must be kept at level l. With no near-tie at any level
    there is one branch, so the row is admissible exactly when it equals ``select_blocks``'s.
    Returns (admissible, reason when not).
    """
    n_levels = len(levels)
    n0 = levels[0].shape[0]
    if budgets is None:
        budgets = [topk] * n_levels
    forced = [] if forced is None else list(forced)
    row = [int(x) for x in row]
    n_valid = next((t for t, x in enumerate(row) if x < 0), len(row))
    valid = row[:n_valid]
    if any(x >= 0 for x in row[n_valid:]):
        return False, "a block after the -1 padding"
    if any(valid[t] >= valid[t + 1] for t in range(len(valid) - 1)):
        return False, "blocks not strictly ascending (unsorted or repeated)"
    if any(j > last or j >= n0 for j in valid):
        return False, "a block that is not eligible"
    if any(f not in valid for f in forced):
        return False, "a forced block is missing"
    target = set(valid) - set(forced)
    top = n_levels - 1
    start = [c for c in range(levels[top].shape[0]) if node_span(n0, factor, top, c)[0] <= last]
    stack = [(top, start)]
    explored = 0
    while stack:
        l, cands = stack.pop()
        explored += 1
        if explored > max_branches:
            return False, "more near-tie branches than the search allows"
        if l == 0 and forced:
            cands = [c for c in cands if c not in forced]
        need = {j // factor ** l for j in target}
        if not need <= set(cands):
            continue
        k_l = budgets[l] - (len(forced) if l == 0 else 0)
        if k_l <= 0:
            options = [[]]
        elif len(cands) <= k_l:
            options = [list(cands)]
        else:
            sc = {c: float(score(qbar, node_value(levels, factor, l, c, last))) for c in cands}
            order = sorted(cands, key=lambda c: rank_key(sc[c], c))
            s_k, s_k1 = sc[order[k_l - 1]], sc[order[k_l]]
            band = []
            if _near(s_k, s_k1, rel_tol):
                band = [c for c in order if _near(sc[c], s_k, rel_tol) or _near(sc[c], s_k1, rel_tol)]
            sure = [c for c in order[:k_l] if c not in band]
            free = k_l - len(sure)
            if not (need - set(band)) <= set(sure):
                continue
            must = [c for c in band if c in need]
            rest = [c for c in band if c not in need]
            if len(must) > free:
                continue
            if l == 0:
                options = [sure + must] if len(must) == free else []
            else:
                if math.comb(len(rest), free - len(must)) > max_branches:
                    return False, "more near-tie branches than the search allows"
                options = [sure + must + list(extra) for extra in itertools.combinations(rest, free - len(must))]
        for kept in options:
            if l == 0:
                if set(kept) == target:
                    return True, ""
                continue
            n_below = levels[l - 1].shape[0]
            nxt = sorted(ch for c in kept for ch in children(n_below, factor, c)
                         if node_span(n0, factor, l - 1, ch)[0] <= last)
            stack.append((l - 1, nxt))
    return False, "no resolution of the near-ties at the pruning levels gives this row"


# ----------------------------------------------------------------------------- attention

def attend(q_rows: np.ndarray, q_pos: np.ndarray, k_plane: np.ndarray, v_plane: np.ndarray,
           blocks: list[int], block: int, causal: bool, scale: float) -> tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of query rows over the keys of the selected blocks (fp32).

    S = scale * q . k for every key of every selected block, keys after the
    query position masked when causal; O = softmax(S) V; LSE = log sum exp S.
    Returns O [R, D] and LSE [R]. A row with no selected block has no key to
    attend to: O = 0 and LSE = -inf (the library's convention for that case).
    """
    if len(blocks) == 0:
        return (np.zeros((q_rows.shape[0], v_plane.shape[1]), dtype=F32),
                np.full(q_rows.shape[0], -np.inf, dtype=F32))
    key_pos = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks])
    kx = k_plane[key_pos].astype(F32)
    vx = v_plane[key_pos].astype(F32)
    s = F32(scale) * (q_rows.astype(F32) @ kx.T)
    if causal:
        s = np.where(key_pos[None, :] > q_pos[:, None], F32(-np.inf), s)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m, dtype=F32)
    l_sum = p.sum(axis=1, keepdims=True, dtype=F32)
    o = (p @ vx) / l_sum
    lse = (m + np.log(l_sum)).reshape(-1)
    return o.astype(F32), lse.astype(F32)


def dense_attention(q_rows: np.ndarray, q_pos: np.ndarray, k_plane: np.ndarray, v_plane: np.ndarray,
                    causal: bool, scale: float, allowed: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """fp64 brute-force softmax attention over all keys (QK^T -> softmax -> V).

    `allowed` [R, N] optionally restricts each row to a subset of keys (-inf elsewhere).
    """
    q = q_rows.astype(np.float64)
    k = k_plane.astype(np.float64)
    v = v_plane.astype(np.float64)
    s = scale * (q @ k.T)
    mask = np.ones_like(s, dtype=bool)
    if causal:
        mask &= np.arange(k.shape[0])[None, :] <= q_pos[:, None]
    if allowed is not None:
        mask &= allowed
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l_sum = p.sum(axis=1, keepdims=True)
    return (p @ v) / l_sum, (m + np.log(l_sum)).reshape(-1)


def merge_partials(outs: list[np.ndarray], lses: list[np.ndarray]) -> tuple[np.ndarray, np.ndarray]:
    """Online-softmax merge of normalised partial attentions over disjoint key sets.

    lse = log sum_i exp(lse_i);  o = sum_i exp(lse_i - lse) o_i.
    """
    lse_stack = np.stack([x.astype(np.float64) for x in lses])
    m = lse_stack.max(axis=0)
    w = np.exp(lse_stack - m)
    total = w.sum(axis=0)
    lse = m + np.log(total)
    o = sum(w[i][:, None] * outs[i].astype(np.float64) for i in range(len(outs))) / total[:, None]
    return o, lse


# ----------------------------------------------------------------------------- backward

def attend_backward(q_rows: np.ndarray, q_pos: np.ndarray, k_plane: np.ndarray, v_plane: np.ndarray,
                    blocks: list[int], block: int, causal: bool, scale: float, d_out: np.ndarray
                    ) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of ``attend`` (fp64) through a fixed selection: the selection itself has no
    gradient (it is a discrete choice), the softmax over the selected keys does.

    With S = scale Q K_sel^T (masked), P = softmax(S) row by row and O = P V_sel:
      dV_sel = P^T dO,  dP = dO V_sel^T,  dS = P * (dP - rowsum(dO * O)),
      dQ = scale dS K_sel,  dK_sel = scale dS^T Q.
    Returns dQ [R, D] and dK, dV over the whole plane [N, D] (zero outside the selected keys).
    """
    dq = np.zeros(q_rows.shape, dtype=np.float64)
    dk = np.zeros(k_plane.shape, dtype=np.float64)
    dv = np.zeros(v_plane.shape, dtype=np.float64)
    if len(blocks) == 0:
        return dq, dk, dv
    key_pos = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks])
    q = q_rows.astype(np.float64)
    kx = k_plane[key_pos].astype(np.float64)
    vx = v_plane[key_pos].astype(np.float64)
    do = d_out.astype(np.float64)
    s = scale * (q @ kx.T)
    if causal:
        s = np.where(key_pos[None, :] > q_pos[:, None], -np.inf, s)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)
    o = p @ vx
    dvx = p.T @ do
    dp = do @ vx.T
    ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
    dq = scale * (ds @ kx)
    np.add.at(dk, key_pos, scale * (ds.T @ q))
    np.add.at(dv, key_pos, dvx)
    return dq, dk, dv


def backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray, idx: np.ndarray, block: int,
             causal: bool, scale: float | None = None, per_qhead: bool = False) -> dict:
    """dQ, dK, dV (fp64) of the sparse attention step for given selected blocks `idx`
    [B, Hsel, nqb, K] (prefill): per query block and head, ``attend_backward``; a KV head's
    dK and dV sum the contributions of all its query heads (GQA)."""
    B, Hq, N, D = Q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    sc = default_scale(D, scale)
    nqb = N // block
    dQ = np.zeros(Q.shape, dtype=np.float64)
    dK = np.zeros(K.shape, dtype=np.float64)
    dV = np.zeros(V.shape, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kvh = h // g
            hs = h if per_qhead else kvh
            for i in range(nqb):
                rows = np.arange(i * block, (i + 1) * block)
                blocks = [int(j) for j in idx[b, hs, i] if j >= 0]
                dq, dk, dv = attend_backward(Q[b, h, rows], rows, K[b, kvh], V[b, kvh], blocks, block, causal,
                                             sc, dO[b, h, rows])
                dQ[b, h, rows] = dq
                dK[b, kvh] += dk
                dV[b, kvh] += dv
    return {"dQ": dQ, "dK": dK, "dV": dV}


# ----------------------------------------------------------------------------- whole forward

def default_scale(head_dim: int, scale: float | None) -> float:
    return 1.0 / math.sqrt(head_dim) if scale is None or scale <= 0 else float(scale)


def selection_heads(heads_q: int, heads_kv: int, per_qhead: bool, hs: int) -> tuple[int, list[int]]:
    """(KV head, query heads) of selection row hs: a KV head's g query heads, or one query head."""
    g = heads_q // heads_kv
    if per_qhead:
        return hs // g, [hs]
    return hs, list(range(hs * g, (hs + 1) * g))


def forward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, block: int, factor: int, topk: int,
            causal: bool, scale: float | None = None, per_qhead: bool = False,
            budgets: list[int] | None = None, idx_override: np.ndarray | None = None,
            forced: int = 0, kv_len: int | None = None) -> dict:
    """Pyramid -> query summaries -> descent top-K -> sparse attention, for whole tensors.

    Q [B, Hq, Nq, D] (Nq = N for prefill, 1 for decode at position N-1), K, V
    [B, Hkv, N, D], all bf16-exact fp32. Selection is shared by the g query heads
    of a KV head unless per_qhead. `idx_override` replaces the oracle's own
    selection in the attention step (used to check attention on given indices).
    Decode over a cache with spare capacity (R17): K and V hold `kv_len` keys
    followed by unused rows; the pyramid has the capacity's levels and the query
    sits at position kv_len - 1.
    """
    B, Hq, Nq, D = Q.shape
    Hkv, N_rows = K.shape[1], K.shape[2]
    N = N_rows if kv_len is None else kv_len
    g = Hq // Hkv
    decode = Nq == 1
    assert kv_len is None or decode, "spare KV capacity is a decode feature"
    sc = default_scale(D, scale)
    n0 = N // block
    hsel = Hq if per_qhead else Hkv
    nqb = 1 if decode else Nq // block
    if kv_len is None:
        pyr = [[build_pyramid(K[b, h], block, factor) for h in range(Hkv)] for b in range(B)]
    else:
        pyr = [[build_pyramid_capacity(K[b, h], block, factor, kv_len) for h in range(Hkv)] for b in range(B)]
    idx = np.full((B, hsel, nqb, topk), -1, dtype=np.int32)
    margin = np.full((B, hsel, nqb), np.inf, dtype=np.float64)
    n_scored = np.zeros((B, hsel, nqb), dtype=np.int64)
    qbars = np.zeros((B, hsel, nqb, D), dtype=F32)
    for b in range(B):
        for hs in range(hsel):
            kvh, heads = selection_heads(Hq, Hkv, per_qhead, hs)
            qbar = query_summary(Q[b, heads], 1 if decode else block)
            qbars[b, hs] = qbar
            for i in range(nqb):
                last = n0 - 1 if (decode or not causal) else i
                fset = forced_set(forced, n0 - 1 if decode else i, topk)
                r = select_blocks(qbar[i], pyr[b][kvh], factor, topk, last, budgets, fset)
                idx[b, hs, i, :len(r["idx"])] = r["idx"]
                margin[b, hs, i] = r["margin"]
                n_scored[b, hs, i] = r["n_scored"]
    use = idx if idx_override is None else idx_override
    O = np.zeros((B, Hq, Nq, D), dtype=F32)
    lse = np.zeros((B, Hq, Nq), dtype=F32)
    for b in range(B):
        for h in range(Hq):
            kvh = h // g
            hs = h if per_qhead else kvh
            for i in range(nqb):
                rows = np.arange(Nq) if decode else np.arange(i * block, (i + 1) * block)
                q_pos = np.full(1, N - 1) if decode else rows
                blocks = [int(j) for j in use[b, hs, i] if j >= 0]
                o, ls = attend(Q[b, h, rows], q_pos, K[b, kvh], V[b, kvh], blocks, block,
                               causal and not decode, sc)
                O[b, h, rows] = o
                lse[b, h, rows] = ls
    return {"O": O, "lse": lse, "idx": idx, "margin": margin, "n_scored": n_scored, "pyramid": pyr,
            "qbar": qbars}
