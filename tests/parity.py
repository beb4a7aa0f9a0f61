"""Helpers that compare the CUDA library's step with the fp64 oracle.

Tolerances (stated for the decode step's outputs): fp32 inputs
|gpu - oracle| <= 1e-5 + 1e-5 |oracle|; bf16 inputs <= 2e-3 + 2e-2 |oracle|.
Selected sets: with tau the oracle's k_eff-th largest selection key, the GPU
set must hold k_eff distinct ascending indices, contain every index whose key
exceeds tau + 1e-3, hold none whose key is below tau - 1e-3, and pad with -1.
Layers are checked with teacher forcing: layer l of the oracle inherits the
GPU's own sets after layer l-1, so one near-tie cannot cascade.  Under the
other selection rules (check_set_rule) a set's size is accepted within the
bands below, and its rows must be a valid choice of that many largest keys.
"""
from __future__ import annotations

import numpy as np

import oracle as O
from hybrid_head_sparse_b200 import workloads as W

TOL = {"fp32": (1e-5, 1e-5), "bf16": (2e-3, 2e-2)}
TIE_BAND = 1e-3


def check_set(gpu_set: np.ndarray, keys: np.ndarray, k: int, what: str):
    n = keys.size
    keff = min(k, n)
    assert gpu_set.shape == (k,)
    assert np.all(gpu_set[keff:] == -1), f"{what}: padding is not -1"
    sel = gpu_set[:keff]
    assert np.all(sel >= 0) and np.all(sel < n), f"{what}: index out of range"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    if keff == n:
        return
    tau = np.sort(keys)[::-1][keff - 1]
    must = np.nonzero(keys > tau + TIE_BAND)[0]
    mustnt = set(np.nonzero(keys < tau - TIE_BAND)[0].tolist())
    s = set(sel.tolist())
    missing = [i for i in must.tolist() if i not in s]
    wrong = [i for i in sel.tolist() if i in mustnt]
    assert not missing, f"{what}: {len(missing)} clearly-selected indices missing, e.g. {missing[:5]}"
    assert not wrong, f"{what}: {len(wrong)} clearly-unselected indices chosen, e.g. {wrong[:5]}"


# Selection rules: a set size decided by probability mass or threshold is
# accepted when the fp64 probabilities put the boundary within MASS_BAND
# (absolute, for top-p's running mass) or PROB_BAND (relative, for a
# threshold) of it; block scores within SCORE_BAND (relative).
MASS_BAND = 2e-3
PROB_BAND = 1e-2
SCORE_BAND = 1e-3


def _valid_prefix(gpu_set: np.ndarray, n: int, what: str) -> np.ndarray:
    m = int(np.argmax(gpu_set < 0)) if np.any(gpu_set < 0) else gpu_set.size
    sel = gpu_set[:m]
    assert np.all(gpu_set[m:] == -1), f"{what}: entries after the padding"
    assert np.all(sel < n), f"{what}: index out of range"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    return sel


def _check_topm(sel: np.ndarray, keys: np.ndarray, what: str):
    """sel (ascending) must be a valid set of the len(sel) largest keys."""
    m = sel.size
    if m == keys.size or m == 0:
        return
    tau = np.sort(keys)[::-1][m - 1]
    s = set(sel.tolist())
    missing = [i for i in np.nonzero(keys > tau + TIE_BAND)[0].tolist() if i not in s]
    wrong = [i for i in sel.tolist() if keys[i] < tau - TIE_BAND]
    assert not missing, f"{what}: {len(missing)} clearly-selected indices missing"
    assert not wrong, f"{what}: {len(wrong)} clearly-unselected indices chosen"


def check_set_rule(gpu_set: np.ndarray, keys: np.ndarray, k: int, sel, what: str):
    """A GPU set against the oracle's fp64 keys under a selection rule
    (oracle.Selection, None = top-k)."""
    n = keys.size
    if sel is None or sel.rule == O.RULE_TOPK:
        return check_set(gpu_set, keys, k, what)
    assert gpu_set.shape == (k,)
    if sel.rule == O.RULE_RATIO:
        num, den = sel.ratio
        m = max(1, min(-((-num * n) // den), k, n))
        assert np.all(gpu_set[m:] == -1), f"{what}: ratio set longer than {m}"
        return check_set(gpu_set[:m], keys, m, what)
    got = _valid_prefix(gpu_set, n, what)
    e = np.exp(keys - keys.max())
    A = e / e.sum()
    if sel.rule == O.RULE_BLOCK_TOPK:
        bs = sel.block
        blocks = np.unique(got // bs)
        rows = [i for b in blocks for i in range(b * bs, min(n, (b + 1) * bs))]
        assert got.tolist() == rows, f"{what}: the set is not made of whole blocks"
        starts = np.arange(0, n, bs)
        score = np.log(np.add.reduceat(A, starts))
        kb = min(k // bs, starts.size)
        assert blocks.size == kb, f"{what}: {blocks.size} blocks, expected {kb}"
        _check_topm_band(blocks, score, SCORE_BAND, what)
        return
    m = got.size
    cap = min(k, n)
    if sel.rule == O.RULE_TOPP:
        cum = np.cumsum(np.sort(A)[::-1])
        lo = int(np.searchsorted(cum, sel.p - MASS_BAND)) + 1
        hi = int(np.searchsorted(cum, sel.p + MASS_BAND)) + 1
    else:
        lo = int((A >= sel.tau * (1 + PROB_BAND)).sum())
        hi = int((A >= sel.tau * (1 - PROB_BAND)).sum())
    lo, hi = min(max(lo, 1), cap), min(max(hi, 1), cap)
    assert lo <= m <= hi, f"{what}: set of {m} rows, expected {lo}..{hi}"
    _check_topm(got, keys, what)


def _check_topm_band(sel: np.ndarray, score: np.ndarray, band: float, what: str):
    m = sel.size
    if m == score.size:
        return
    tau = np.sort(score)[::-1][m - 1]
    s = set(sel.tolist())
    missing = [i for i in np.nonzero(score > tau + band)[0].tolist() if i not in s]
    wrong = [i for i in sel.tolist() if score[i] < tau - band]
    assert not missing and not wrong, f"{what}: block choice off ({len(missing)} missing, {len(wrong)} wrong)"


def check_out(gpu: np.ndarray, ora: np.ndarray, dtype: str, what: str):
    atol, rtol = TOL[dtype]
    err = np.abs(gpu.astype(np.float64) - ora)
    bound = atol + rtol * np.abs(ora)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs off; "
                           f"max err {err.max():.3e} (bound there {bound.flat[err.argmax()]:.3e})")
    return float(err.max())


def host_stack(data: dict, layers=None, select_mode=O.SELECT_PER_QHEAD) -> O.Stack:
    """Host copy of the step's inputs (optionally only some layers)."""
    q, K, V = data["q"], data["k"], data["v"]
    role = data["role"]
    if layers is not None:
        idx = list(layers)
        q, K, V, role = q[idx], K[idx], V[idx], role[idx]
    return O.Stack(W.host_view(q), W.host_view(K), W.host_view(V),
                   np.ascontiguousarray(role, dtype=np.uint8), select_mode)


def check_layers(data: dict, out, trace: np.ndarray, k: int, n: int, dtype: str,
                 layers, select_mode=O.SELECT_PER_QHEAD, S0: np.ndarray | None = None, sel=None):
    """Check the chosen layers of a GPU step (out [L][B][Hq][d], or a list of
    such arrays from runs that inherited the same sets; trace [L][B][Hs][k])
    against the oracle with teacher forcing.  S0: the sets handed to layer 0
    (set-input mode) or None (layer 0 all retrieval)."""
    outs = out if isinstance(out, (list, tuple)) else [out]
    worst = 0.0
    for l in layers:
        st = host_stack(data, layers=[l], select_mode=select_mode)
        if l == 0:
            S_in = S0
            all_ret = S0 is None
        else:
            S_in = trace[l - 1]
            all_ret = False
        o, S_out, keys, fresh = O.layer(st, 0, k, S_in, all_retrieval=all_ret, n=n, sel=sel)
        for i, ou in enumerate(outs):
            worst = max(worst, check_out(ou[l], o, dtype, f"layer {l} outputs (run {i})"))
        B, Hs = S_out.shape[:2]
        for b in range(B):
            for s in range(Hs):
                if fresh[s]:
                    check_set_rule(trace[l, b, s], keys[b, s], k, sel, f"layer {l} b {b} set {s}")
                else:
                    assert np.array_equal(trace[l, b, s], S_in[b, s]), \
                        f"layer {l} b {b} set {s}: an unrefreshed set changed"
    return worst


def check_layers_varlen(q: np.ndarray, K: np.ndarray, V: np.ndarray, role: np.ndarray,
                        n_list, out: np.ndarray, trace: np.ndarray, k: int, dtype: str, layers,
                        select_mode=O.SELECT_PER_QHEAD, S0: np.ndarray | None = None, sel=None):
    """The serving form: element b of the batch is checked on its own, as a
    one-element step over its n[b] rows (the logical cache after the append),
    with teacher forcing as in check_layers.  q [L][B][Hq][d], K/V
    [L][B][Hkv][rows][d] host arrays (bf16 as uint16 bit patterns)."""
    worst = 0.0
    for b, nb in enumerate(n_list):
        for l in layers:
            st = O.Stack(np.ascontiguousarray(q[l:l + 1, b:b + 1]),
                         np.ascontiguousarray(K[l:l + 1, b:b + 1, :, :nb]),
                         np.ascontiguousarray(V[l:l + 1, b:b + 1, :, :nb]),
                         np.ascontiguousarray(role[l:l + 1], dtype=np.uint8), select_mode)
            if l == 0:
                S_in = None if S0 is None else S0[b:b + 1]
                all_ret = S0 is None
            else:
                S_in = trace[l - 1, b:b + 1]
                all_ret = False
            o, S_out, keys, fresh = O.layer(st, 0, k, S_in, all_retrieval=all_ret, sel=sel)
            worst = max(worst, check_out(out[l, b:b + 1], o, dtype, f"b {b} layer {l} outputs"))
            for s in range(S_out.shape[1]):
                if fresh[s]:
                    check_set_rule(trace[l, b, s], keys[0, s], k, sel, f"b {b} layer {l} set {s}")
                else:
                    assert np.array_equal(trace[l, b, s], S_in[0, s]), \
                        f"b {b} layer {l} set {s}: an unrefreshed set changed"
    return worst
