"""Planted mistakes in the oracle must each fail at least one pin.

Each mutation patches one oracle function on the CPU with a plausible slip (a
dropped term, a wrong sign, an off-by-one index, a swapped operand) and runs
the pins; the test passes when some pin raises. This shows the pins can see
mistakes in every step, not only that the current oracle passes them.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import pisa_oracle as po
from tests import pins

F32 = np.float32
_orig_children = po.children
_orig_block_means = po.block_means
_orig_attend = po.attend
_orig_node_value = po.node_value
_orig_query_summary = po.query_summary
_orig_merge = po.merge_partials
_orig_level_sizes = po.level_sizes
_orig_attend_backward = po.attend_backward


def _drop_last_child(n_below, factor, c):
    return list(range(c * factor, min(c * factor + factor - 1, n_below)))


def _mean_off_by_one(k_plane, block):
    n0 = k_plane.shape[0] // block
    return k_plane[:n0 * block].astype(F32).reshape(n0, block, -1).sum(axis=1) / F32(block + 1)


def _rank_ascending(score_value, node):
    return (float(score_value), node)


def _rank_ties_high(score_value, node):
    return (-float(score_value), -node)


def _attend_causal_strict(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale):
    return _orig_attend(q_rows, q_pos - 1, k_plane, v_plane, blocks, block, causal, scale)


def _attend_no_scale(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale):
    return _orig_attend(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, 1.0)


def _attend_values_swapped(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale):
    return _orig_attend(q_rows, q_pos, v_plane, k_plane, blocks, block, causal, scale)


def _node_value_leaky(levels, factor, level, c, last):
    return levels[level][c]


def _query_first_head(q_heads, rows_per_block):
    return _orig_query_summary(q_heads[:1], rows_per_block)


def _merge_wrong_sign(outs, lses):
    return _orig_merge(outs, [-x for x in lses])


def _score_dropped_component(qbar, node):
    return F32(np.dot(qbar[1:].astype(F32), node[1:].astype(F32)))


def _forced_not_truncated(forced, local, topk):
    out = [0] if forced & 1 else []
    if forced & 2 and local not in out:
        out.append(local)
    return out


def _forced_repeats_sink(forced, local, topk):
    out = [0] if forced & 1 else []
    if forced & 2:
        out.append(local)
    return out[:topk]


def _forced_local_is_previous_block(forced, local, topk):
    out = [0] if forced & 1 else []
    if forced & 2 and max(local - 1, 0) not in out:
        out.append(max(local - 1, 0))
    return out[:topk]


def _capacity_counts_spare_blocks(k_plane, block, factor, kv_len):
    return po.build_pyramid(k_plane, block, factor)


def _backward_no_delta(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale, d_out):
    # dS = P * dP (the row term rowsum(dO * O) dropped) is what dQ and dK then carry
    dq, dk, dv = _orig_attend_backward(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale, d_out)
    dq2, dk2, dv2 = _orig_attend_backward(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale,
                                          np.zeros_like(d_out))
    key_pos = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks]) if blocks else []
    if len(key_pos) == 0:
        return dq, dk, dv
    q = q_rows.astype(np.float64)
    kx = k_plane[key_pos].astype(np.float64)
    vx = v_plane[key_pos].astype(np.float64)
    s = scale * (q @ kx.T)
    if causal:
        s = np.where(np.asarray(key_pos)[None, :] > q_pos[:, None], -np.inf, s)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ds = p * (d_out.astype(np.float64) @ vx.T)
    dk_bad = np.zeros_like(dk)
    np.add.at(dk_bad, key_pos, scale * (ds.T @ q))
    return scale * (ds @ kx), dk_bad, dv


def _backward_dk_unscaled(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale, d_out):
    dq, dk, dv = _orig_attend_backward(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale, d_out)
    return dq, dk / scale, dv


def _backward_with_slip(slip):
    """The oracle's backward restated with one planted slip."""
    def bad(q_rows, q_pos, k_plane, v_plane, blocks, block, causal, scale, d_out):
        if slip == "no_mask":
            return _orig_attend_backward(q_rows, q_pos, k_plane, v_plane, blocks, block, False, scale, d_out)
        dq = np.zeros(q_rows.shape)
        dk = np.zeros(k_plane.shape)
        dv = np.zeros(v_plane.shape)
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
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ vx
        dp = do @ vx.T
        ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
        dvx = (ds if slip == "dv_from_ds" else p).T @ do
        dq = scale * (ds @ (vx if slip == "dq_from_v" else kx))
        np.add.at(dk, key_pos, scale * (ds.T @ q))
        np.add.at(dv, key_pos, dvx)
        return dq, dk, dv
    return bad


def _one_level_too_many(n0, factor):
    sizes = [n0]
    while sizes[-1] >= factor:
        sizes.append(-(-sizes[-1] // factor))
    return sizes


MUTATIONS = {
    "pyramid drops a child": ("children", _drop_last_child),
    "level-0 mean divides by block+1": ("block_means", _mean_off_by_one),
    "selection keeps the lowest scores": ("rank_key", _rank_ascending),
    "ties go to the higher index": ("rank_key", _rank_ties_high),
    "causal mask excludes the diagonal key": ("attend", _attend_causal_strict),
    "softmax scale dropped": ("attend", _attend_no_scale),
    "K and V swapped": ("attend", _attend_values_swapped),
    "straddling node leaks future keys": ("node_value", _node_value_leaky),
    "query summary uses one head of the group": ("query_summary", _query_first_head),
    "merge weights with the wrong sign": ("merge_partials", _merge_wrong_sign),
    "score drops one component": ("score", _score_dropped_component),
    "pyramid builds one level too many": ("level_sizes", _one_level_too_many),
    "forced blocks exceed K": ("forced_set", _forced_not_truncated),
    "sink repeated as the local block": ("forced_set", _forced_repeats_sink),
    "local block off by one": ("forced_set", _forced_local_is_previous_block),
    "capacity pyramid averages the spare rows": ("build_pyramid_capacity", _capacity_counts_spare_blocks),
    "backward drops the row term of dS": ("attend_backward", _backward_no_delta),
    "backward leaves the scale out of dK": ("attend_backward", _backward_dk_unscaled),
    "backward ignores the causal mask": ("attend_backward", _backward_with_slip("no_mask")),
    "backward forms dV from dS instead of P": ("attend_backward", _backward_with_slip("dv_from_ds")),
    "backward multiplies dS by V for dQ": ("attend_backward", _backward_with_slip("dq_from_v")),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(po, attr, bad)
    failed = []
    for pin_name, pin in pins.ALL_PINS.items():
        try:
            pin(po)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin_name)
    assert failed, f"no pin caught: {name}"


def test_restated_backward_without_a_slip_passes(monkeypatch):
    """Control for the backward slips above: the same restatement with no slip passes every pin,
    so what those mutations trip is the slip, not the restatement."""
    monkeypatch.setattr(po, "attend_backward", _backward_with_slip("none"))
    for pin_name, pin in pins.ALL_PINS.items():
        if pin_name.startswith("backward"):
            pin(po)
